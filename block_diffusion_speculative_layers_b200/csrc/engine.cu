// engine.cu -- the dflash C ABI: configuration checks, arena layout, weight
// slots and the orchestration of prefill, draft, verify+commit and whole
// generations.  Every step of the path runs in the kernels of this library;
// the host only launches them and checks arguments.
//
// The decode iteration follows the DFlash pages (by title and section):
//  * "DFlash: Decodificação Especulativa com Blocos em Paralelo ..." (iaemfoco):
//    "O que o DFlash faz de diferente" -- one drafter pass proposes the whole
//    block, one target pass verifies it; "O alvo sabe mais" -- hidden states
//    of several target layers are fused into a context vector and injected
//    into the Key/Value projections of every drafter layer (persisting in the
//    drafter KV cache); "Decodificação especulativa tradicional" -- lossless.
//  * "DFlash e Spec V2 revolucionam a speculative decoding" (ceviu): host-device
//    synchronisation kept to the minimum -> the whole iteration is enqueued
//    without host round trips; generate() polls a done counter once per
//    iteration, one iteration behind.
#include <algorithm>
#include <chrono>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>
#include <type_traits>

#include "engine.h"
#include "gemm_tc.h"
#include "attn_mma.h"
#include "attn_tma.h"
#include "pass_program.h"

namespace dfl {

// Scratch of dflash_head_argmax_noalloc: per-(vocab tile, row) partial maxima
// for up to 64 rows and 2048 vocab tiles (vocab <= 262144), then the output ids.
constexpr int kNoallocRows = 64;
constexpr int kNoallocTiles = 2048;
constexpr size_t kNoallocPartBytes = (size_t)kNoallocRows * kNoallocTiles * sizeof(float2);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocPartBytes + kNoallocRows * sizeof(int)];

// Device address of g_noalloc_scratch on device `dev` (the host-side symbol is
// not a device address), looked up once per device with that device current,
// under a lock so that host threads driving different contexts can share it.
static void *noalloc_scratch_ptr(int dev, std::string &err) {
    static std::mutex mu;
    static void *ptrs[kMaxDevices] = {nullptr};
    if (dev < 0 || dev >= kMaxDevices) {
        err = "device index out of range";
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        int prev = 0;
        if (cudaGetDevice(&prev) != cudaSuccess) {
            err = "no current CUDA device";
            return nullptr;
        }
        void *p = nullptr;
        cudaError_t e = cudaSetDevice(dev);
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        cudaSetDevice(prev);
        if (e != cudaSuccess) {
            err = std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
            return nullptr;
        }
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static int elem_size(int dtype) {
    return dtype == DFLASH_FP32 ? 4 : (dtype == DFLASH_FP8 || dtype == DFLASH_FP4 || dtype == DFLASH_UE8M0) ? 1 : 2;
}

static bool check_model(const dflash_model_cfg &m, std::string &why) {
    if (m.n_layers < 1 || m.hidden < 32 || m.n_q_heads < 1 || m.n_kv_heads < 1 || m.vocab < 2) {
        why = "model dimensions must be positive";
        return false;
    }
    if (m.n_q_heads % m.n_kv_heads) { why = "n_q_heads must be a multiple of n_kv_heads"; return false; }
    if (m.n_q_heads / m.n_kv_heads > 8) { why = "at most 8 q heads per kv head"; return false; }
    if (m.head_dim != 64 && m.head_dim != 128) { why = "head_dim must be 64 or 128"; return false; }
    if (m.hidden % 64) { why = "hidden must be a multiple of 64"; return false; }
    if (m.n_experts < 0 || m.n_experts > 256) { why = "n_experts must be in [0, 256]"; return false; }
    if (m.n_experts > 0) {
        if (m.top_k < 1 || m.top_k > m.n_experts || m.top_k > 32 || m.expert_ffn < 8 || m.expert_ffn % 8) {
            why = "bad MoE dims (top_k in [1, min(E,32)], expert_ffn multiple of 8)";
            return false;
        }
    } else if (m.ffn < 8 || m.ffn % 8) {
        why = "ffn must be a positive multiple of 8";
        return false;
    }
    if (!(m.rms_eps >= 0.0) || !(m.rope_theta > 1.0)) { why = "bad rms_eps / rope_theta"; return false; }
    if (m.n_q_heads + m.n_kv_heads > 256) { why = "at most 256 q + kv heads"; return false; }
    if (m.qk_norm != 0 && m.qk_norm != 1) { why = "qk_norm must be 0 or 1"; return false; }
    if (m.rope_factor > 1.0 && !(m.rope_low_freq_factor > 0.0 && m.rope_high_freq_factor > m.rope_low_freq_factor &&
                                 m.rope_original_max_pos > 0.0)) {
        why = "RoPE rescaling needs 0 < low < high and original_max_pos > 0";
        return false;
    }
    return true;
}

static bool check_config(const dflash_config &c, std::string &why) {
    if (!check_model(c.target, why)) { why = "target: " + why; return false; }
    if (!check_model(c.drafter, why)) { why = "drafter: " + why; return false; }
    if (c.drafter.n_experts != 0) { why = "the drafter must be dense"; return false; }
    if (c.drafter.hidden != c.target.hidden || c.drafter.vocab != c.target.vocab) {
        why = "drafter hidden/vocab must equal the target's (shared embedding and head)";
        return false;
    }
    if (c.block_size < 1 || c.block_size > DFLASH_MAX_BLOCK) { why = "block_size must be in [1, 32]"; return false; }
    if (c.n_taps < 1 || c.n_taps > DFLASH_MAX_TAPS) { why = "n_taps must be in [1, 8]"; return false; }
    for (int i = 0; i < c.n_taps; ++i)
        if (c.tap_layers[i] < 0 || c.tap_layers[i] >= c.target.n_layers) { why = "tap layer out of range"; return false; }
    if (c.mask_token_id < 0 || c.mask_token_id >= c.target.vocab) { why = "mask_token_id out of vocab"; return false; }
    if (c.max_batch < 1 || c.max_batch > 64) { why = "max_batch must be in [1, 64]"; return false; }
    if (c.max_len < c.block_size + 1 || c.max_len > (1 << 20)) { why = "max_len out of range"; return false; }
    if (c.prefill_chunk < 0 || c.prefill_chunk > 8192) { why = "prefill_chunk must be in [0, 8192]"; return false; }
    if (c.dtype != DFLASH_FP32 && c.dtype != DFLASH_BF16 && c.dtype != DFLASH_BF16_FAST && c.dtype != DFLASH_FP8 &&
        c.dtype != DFLASH_FP4) {
        why = "dtype must be DFLASH_FP32, DFLASH_BF16, DFLASH_BF16_FAST, DFLASH_FP8 or DFLASH_FP4";
        return false;
    }
    if (c.dtype == DFLASH_FP4) {
        // MXFP4 rows: K (hidden, ffn, q width, n_taps * hidden) in whole 128-value groups
        const dflash_model_cfg *ms[2] = {&c.target, &c.drafter};
        for (const dflash_model_cfg *m : ms) {
            if (m->n_experts > 0) { why = "FP4 weights need dense models"; return false; }
            if (m->hidden % 128 || m->ffn % 128 || (m->n_q_heads * m->head_dim) % 128) {
                why = "FP4 weights need hidden, ffn and q width multiples of 128";
                return false;
            }
        }
    }
    if (c.dtype == DFLASH_FP8) {
        const dflash_model_cfg *ms[2] = {&c.target, &c.drafter};
        for (const dflash_model_cfg *m : ms) {
            if (m->n_experts > 0) { why = "FP8 weights need dense models"; return false; }
            if (m->hidden % 16 || m->ffn % 16 || (m->n_q_heads * m->head_dim) % 16) {
                why = "FP8 weights need hidden, ffn and q width multiples of 16";
                return false;
            }
        }
    }
    return true;
}

static void add_slot(Layout &L, const std::string &name, int ndim, int64_t d0, int64_t d1, int64_t d2, int dtype);

// A projection matrix [d0, d1]; FP8 storage adds "<name>.scale" [d0] (fp32, one per
// row); FP4 (MXFP4) stores the codes two per byte [d0, d1/2] and adds
// "<name>.bscale" [d1/128, d0, 4] (UE8M0 block exponents) and "<name>.scale".
static void add_matrix(Layout &L, const std::string &name, int64_t d0, int64_t d1, int dtype) {
    if (dtype == DFLASH_FP4) {
        add_slot(L, name, 2, d0, d1 / 2, 0, DFLASH_FP4);
        add_slot(L, name + ".bscale", 3, d1 / 128, d0, 4, DFLASH_UE8M0);
    } else {
        add_slot(L, name, 2, d0, d1, 0, dtype);
    }
    if (dtype == DFLASH_FP8 || dtype == DFLASH_FP4) add_slot(L, name + ".scale", 1, d0, 0, 0, DFLASH_FP32);
}

static void add_slot(Layout &L, const std::string &name, int ndim, int64_t d0, int64_t d1, int64_t d2, int dtype) {
    WeightSlot s;
    s.name = name;
    s.ndim = ndim;
    s.shape[0] = d0;
    s.shape[1] = d1;
    s.shape[2] = d2;
    s.numel = (size_t)d0 * (ndim > 1 ? d1 : 1) * (ndim > 2 ? d2 : 1);
    s.dtype = dtype;
    L.weight_bytes = align_up(L.weight_bytes, 256);
    s.offset = L.weight_bytes;
    L.weight_bytes += s.numel * elem_size(dtype);
    L.slots.push_back(s);
}

static void add_model_slots(Layout &L, const char *prefix, const dflash_model_cfg &m, int dt) {
    const int64_t H = m.hidden, qd = (int64_t)m.n_q_heads * m.head_dim, kd = (int64_t)m.n_kv_heads * m.head_dim;
    for (int l = 0; l < m.n_layers; ++l) {
        std::string p = std::string(prefix) + ".L" + std::to_string(l) + ".";
        add_slot(L, p + "attn_norm", 1, H, 0, 0, DFLASH_FP32);
        if (m.qk_norm) {
            add_slot(L, p + "q_norm", 1, m.head_dim, 0, 0, DFLASH_FP32);
            add_slot(L, p + "k_norm", 1, m.head_dim, 0, 0, DFLASH_FP32);
        }
        add_matrix(L, p + "wqkv", qd + 2 * kd, H, dt);
        add_matrix(L, p + "wo", H, qd, dt);
        add_slot(L, p + "ffn_norm", 1, H, 0, 0, DFLASH_FP32);
        if (m.n_experts > 0) {
            add_slot(L, p + "w_router", 2, m.n_experts, H, 0, dt);
            add_slot(L, p + "we_gate_up", 3, m.n_experts, 2 * (int64_t)m.expert_ffn, H, dt);
            add_slot(L, p + "we_down", 3, m.n_experts, H, m.expert_ffn, dt);
        } else {
            add_matrix(L, p + "w_gate_up", 2 * (int64_t)m.ffn, H, dt);
            add_matrix(L, p + "w_down", H, m.ffn, dt);
        }
    }
    add_slot(L, std::string(prefix) + ".final_norm", 1, H, 0, 0, DFLASH_FP32);
}

static Layout make_layout(const dflash_config &c) {
    Layout L;
    // weight storage: fp32 or bf16 (both bf16 activation modes store bf16 weights);
    // FP8: every projection matrix as E4M3 codes + row scales, the embedding in bf16
    const int dt_emb = c.dtype == DFLASH_FP32 ? DFLASH_FP32 : DFLASH_BF16, es = elem_size(dt_emb);
    const int dt = (c.dtype == DFLASH_FP8 || c.dtype == DFLASH_FP4) ? c.dtype : dt_emb;
    const dflash_model_cfg &t = c.target, &d = c.drafter;
    add_slot(L, "embed", 2, t.vocab, t.hidden, 0, dt_emb);
    add_matrix(L, "lm_head", t.vocab, t.hidden, dt);
    add_model_slots(L, "target", t, dt);
    add_model_slots(L, "drafter", d, dt);
    add_matrix(L, "fuse.w_fc", d.hidden, (int64_t)c.n_taps * t.hidden, dt);
    add_slot(L, "fuse.norm", 1, d.hidden, 0, 0, DFLASH_FP32);
    L.weight_bytes = align_up(L.weight_bytes, 256);

    const int B = c.block_size, nb = c.max_batch, H = t.hidden;
    L.R_dec = nb * B;
    L.C = c.prefill_chunk > 0 ? c.prefill_chunk : 1024;
    L.R_max = std::max(2 * L.R_dec, L.C);
    const int qd_t = t.n_q_heads * t.head_dim, kd_t = t.n_kv_heads * t.head_dim;
    const int qd_d = d.n_q_heads * d.head_dim, kd_d = d.n_kv_heads * d.head_dim;
    const int F_t = t.n_experts > 0 ? t.expert_ffn : t.ffn;
    int ycols = std::max({qd_t + 2 * kd_t, qd_d + 2 * kd_d, 2 * d.ffn, H});
    if (t.n_experts == 0) ycols = std::max(ycols, 2 * t.ffn);
    else ycols = std::max(ycols, t.n_experts);
    L.Y_cols = ycols;
    const int qmax = std::max(qd_t, qd_d);
    const int fmax = std::max(F_t, d.ffn);
    const int TK = c.n_taps * H;
    const size_t R = L.R_max;
    size_t o = 0;
    auto take = [&](size_t bytes) { o = align_up(o, 256); size_t r = o; o += std::max<size_t>(bytes, 16); return r; };
    // Activations in the model dtype (GEMM inputs, q, the K/V caches) form one
    // contiguous span; with two-plane bf16 activations (DFLASH_BF16) the span is
    // repeated right after itself for the low planes, so every such buffer p has
    // its low plane at p + act_lo elements.
    const size_t act0 = o;
    L.xn = take(R * H * es);
    L.dq_in = take((size_t)2 * L.R_dec * H * es);
    L.q = take(R * qmax * es);
    L.ao = take(R * qmax * es);
    const size_t hrows = t.n_experts > 0 ? R * (size_t)t.top_k : R;
    L.h = take(hrows * fmax * es);
    L.taps_dec = take((size_t)L.R_dec * TK * es);
    L.taps_gather = take((size_t)L.R_dec * TK * es);
    L.taps_pre = take((size_t)L.C * TK * es);
    L.cbuf = take((size_t)L.C * H * es);
    const size_t kv_t = (size_t)t.n_layers * nb * t.n_kv_heads * c.max_len * t.head_dim * es;
    const size_t kv_d = (size_t)d.n_layers * nb * d.n_kv_heads * c.max_len * d.head_dim * es;
    L.tk = take(kv_t);
    L.tv = take(kv_t);
    L.dk = take(kv_d);
    L.dv = take(kv_d);
    L.xg_t = take((size_t)L.R_dec * H * es);
    L.xg2 = take((size_t)L.R_dec * H * es);
    // MoE decode: the pairs' activation rows in expert-grouped order
    L.moe_xg = take(t.n_experts > 0 ? (size_t)L.R_dec * t.top_k * H * es : 16);
    const size_t act_bytes = align_up(o, 256) - act0;
    if (c.dtype == DFLASH_BF16 || c.dtype == DFLASH_FP8 || c.dtype == DFLASH_FP4) {
        take(act_bytes);
        L.act_lo = act_bytes / es;
    }
    L.x = take(R * H * 4);
    L.Y = take(R * (size_t)ycols * 4);
    L.logits = take((size_t)L.R_dec * t.vocab * 4);
    L.plogits = take((size_t)t.vocab * 4);
    {
        // temperature sampling: drafter logits kept through the verify pass, per-row
        // log-sum-exp, chunk partials of the sampling passes, target and residual draws
        const size_t rs = c.sampling ? (size_t)L.R_dec : 0, nc = (size_t)sample_chunks(t.vocab);
        L.qlogits = take(rs * t.vocab * 4);
        L.lse_p = take(rs * 4);
        L.lse_q = take(rs * 4);
        L.samp_part = take(std::max(rs, (size_t)1) * nc * 16);
        L.tok_p = take(rs * 4);
        L.resid = take(rs * 4);
    }
    L.g = take((size_t)L.R_dec * 4);
    L.drafts = take((size_t)nb * B * 4);
    L.accept = take((size_t)nb * 4);
    L.committed = take((size_t)nb * B * 4);
    L.new_len = take((size_t)nb * 4);
    L.st = take((size_t)nb * sizeof(SeqState));
    L.active = take((size_t)nb * 4);
    L.meta = take(R * sizeof(RowMeta));
    L.ctx_meta = take((size_t)L.R_dec * sizeof(RowMeta));
    L.ctx_meta_pre = take((size_t)L.C * sizeof(RowMeta));
    L.rope_t = take((size_t)c.max_len * (t.head_dim / 2) * sizeof(float2));
    L.rope_d = take((size_t)c.max_len * (d.head_dim / 2) * sizeof(float2));
    L.script = take((size_t)nb * c.max_len * 4);
    L.out_tok = take((size_t)nb * c.max_len * 4);
    L.tokens = take((size_t)c.max_len * 4);
    L.stats = take(sizeof(DevStats));
    L.first_tok = take(16);
    const size_t mrows = t.n_experts > 0 ? R * (size_t)t.top_k : 1;
    L.moe_sel = take(mrows * 4);
    L.moe_wt = take(mrows * 4);
    L.moe_part = take(t.n_experts > 0 ? mrows * H * 4 : 16);
    L.moe_off = take(t.n_experts > 0 ? (size_t)(2 * t.n_experts + 2) * 4 : 16);
    L.moe_list = take(mrows * 4);
    // per-(vocab tile, row) best logit of the LM-head GEMM
    L.lm_part = take((size_t)((t.vocab + 127) / 128) * std::max(L.R_dec, 1) * sizeof(float2));
    // split-KV attention partials (sized for 148 SMs; launches cap their splits to fit)
    {
        const int nq_max = std::max(t.n_q_heads, d.n_q_heads), nkv_min = std::min(t.n_kv_heads, d.n_kv_heads);
        const int hd_max = std::max(t.head_dim, d.head_dim);
        const int tiles = std::max(L.R_dec, (L.C + 15) / 16);
        AttnWorkspace aw = attn_workspace_plan(tiles, nq_max, nkv_min, c.max_len, 148);
        L.att_parts = aw.max_parts;
        L.att_o = take(L.att_parts * hd_max * 4);
        L.att_ml = take(L.att_parts * 2 * 4);
        L.att_sem = take((size_t)tiles * std::max(t.n_kv_heads, d.n_kv_heads) * 4);
    }
    // bf16 decode passes: folded-norm activations, per-tile sums of squares and
    // the completion counters of the two pass programs (verify, draft)
    {
        L.ssq_ld = 2 * L.R_dec;
        L.ssq = take((size_t)(H / 128 + 1) * L.ssq_ld * 4);
        L.n_ops_v = 1 + 4 * t.n_layers;
        L.n_ops_d = 2 + 4 * d.n_layers;
        L.dep_v = take((size_t)2 * L.n_ops_v * 4);
        L.dep_d = take((size_t)2 * L.n_ops_d * 4);
    }
    // FP8 / FP4 projections: the activation rows as MX planes (codes + scale words),
    // sized for the most rows and the widest K of any projection
    if (c.dtype == DFLASH_FP8 || c.dtype == DFLASH_FP4) {
        const int kmax = std::max({t.hidden, d.hidden, qmax, fmax, TK});
        L.mx_mpad = (int)align_up((size_t)L.R_max, 32);
        L.mx_kpad = (int)align_up((size_t)kmax, 128);
        L.mx_codes = take((size_t)4 * L.mx_mpad * L.mx_kpad);
        L.mx_words = take((size_t)(L.mx_kpad / 128) * 4 * L.mx_mpad * 4);
    }
    // split-K workspace and tile semaphores of the tensor-core GEMM
    L.ws_floats = gemm_tc_workspace_floats(L.R_max, std::max(ycols, t.vocab > 0 ? H : H));
    L.gemm_ws = take((size_t)L.ws_floats * 4);
    L.n_sem = gemm_tc_semaphores();
    L.gemm_sem = take((size_t)L.n_sem * 4);
    (void)kd_t;
    (void)kd_d;
    L.state_bytes = align_up(o, 256);
    return L;
}

// ------------------------------------------------------------------------
// engine
// ------------------------------------------------------------------------

template <typename T>
class Engine : public EngineBase {
  public:
    dflash_config c;
    const Layout &L;
    cudaStream_t s;
    char *W, *S;
    // weights
    const T *embed;
    const void *lm_head, *w_fc;
    // FP8 / FP4 weights (f8_: either; f4_: MXFP4): the scale vector of every
    // projection matrix and, for FP4, its block exponents and row count, by the
    // matrix's base address
    bool f8_ = false, f4_ = false;
    std::unordered_map<const void *, const float *> wscales;
    std::unordered_map<const void *, std::pair<const uint8_t *, int>> wbscales;
    const float *fc_norm, *t_final, *d_final;
    std::vector<LayerW> tl, dl;
    // state
    float *x, *Y, *logits, *plogits, *moe_wt, *moe_part;
    float *qlogits = nullptr, *lse_p = nullptr, *lse_q = nullptr;
    float4 *samp_part = nullptr;
    int *tok_p = nullptr, *resid = nullptr;
    T *xn, *dq_in, *q, *ao, *h, *taps_dec, *taps_gather, *taps_pre, *cbuf, *tk, *tv, *dk, *dv;
    T *moe_xg = nullptr;
    bool moe_grouped_on = false;  // MoE decode experts as grouped tensor-core projections
    int *g, *drafts, *accept, *committed, *new_len, *active, *script, *out_tok, *tokens, *first_tok, *moe_sel;
    int *moe_off = nullptr, *moe_list = nullptr;
    SeqState *st;
    RowMeta *meta, *ctx_meta, *ctx_meta_pre;
    float2 *rope_t, *rope_d;
    DevStats *stats;
    float *gemm_ws;
    int *gemm_sem;
    float2 *lm_part;
    AttnScratch att;
    // TMA attention: K / V maps of the target (0) and the drafter (1) caches
    AttnTmaMaps kv_map[2];
    bool attn_tma_on = false;
    // folded-norm decode passes (bf16)
    T *xg_t = nullptr, *xg2 = nullptr;
    size_t lo_ = 0;  // low plane offset of two-plane activations (elements), 0: one plane
    float *ssq = nullptr;
    PassProgram pv, pd;
    // bf16 decode passes run as projection programs with folded RMSNorms
    // (fold_*_ok), one kernel per projection
    bool fold_verify_ok = false, fold_draft_ok = false;
    bool dep_on = false;  // completion counters between the kernels of a pass (per-kernel mode)
    bool fold_used[3] = {false, false, false};
    int num_sms = 148;
    GemmTC<T> tc;
    // host mirrors
    std::vector<int> h_len, h_prefilled;
    std::vector<int> last_draft;
    int last_logits_rows[3] = {0, 0, 0};
    // kind of the last pass that ran on this context: what the LM-head input
    // buffers (xn / xg_t) hold now.  PASS_OTHER: generation loops, target-only steps.
    enum { PASS_NONE = -1, PASS_DRAFT = 0, PASS_VERIFY = 1, PASS_PREFILL = 2, PASS_OTHER = 3 };
    int last_pass = PASS_NONE;
    struct OtherPass {  // marks a generation loop on every return path
        int &r;
        ~OtherPass() { r = PASS_OTHER; }
    };
    int device = 0;
    int *pinned = nullptr;  // small pinned host buffer for the done counter
    bool lens_stale = false;
    // per-launch timing (dflash_profile)
    struct ProfRec { int cls[3]; double bytes; cudaEvent_t a, b; };  // classes (-1: none)
    int profiling = 0;  // bit 0: events around every projection / attention launch; bit 1: around passes
    std::vector<ProfRec> prof;
    std::vector<cudaEvent_t> ev_pool;
    size_t ev_used = 0;
    cudaEvent_t ev_a = nullptr, ev_b = nullptr;

    Engine(const dflash_config &cfg, const Layout &lay, char *warena, char *sarena, cudaStream_t stream)
        : c(cfg), L(lay), s(stream), W(warena), S(sarena) {}

    template <typename P>
    P *sp(size_t off) { return reinterpret_cast<P *>(S + off); }

    const void *wslot(const std::unordered_map<std::string, int> &by, const std::string &n) {
        return W + L.slots[by.at(n)].offset;
    }

    dflash_status init(const std::unordered_map<std::string, int> &by) {
        embed = (const T *)wslot(by, "embed");
        lm_head = wslot(by, "lm_head");
        w_fc = wslot(by, "fuse.w_fc");
        f8_ = c.dtype == DFLASH_FP8 || c.dtype == DFLASH_FP4;
        f4_ = c.dtype == DFLASH_FP4;
        auto ends = [](const std::string &s, const char *suf) {
            const size_t n = strlen(suf);
            return s.size() > n && s.compare(s.size() - n, n, suf) == 0;
        };
        if (f8_)
            for (const WeightSlot &sl : L.slots) {
                if (ends(sl.name, ".scale"))
                    wscales[W + L.slots[by.at(sl.name.substr(0, sl.name.size() - 6))].offset] =
                        (const float *)(W + sl.offset);
                if (ends(sl.name, ".bscale"))
                    wbscales[W + L.slots[by.at(sl.name.substr(0, sl.name.size() - 7))].offset] = {
                        (const uint8_t *)(W + sl.offset), (int)sl.shape[1]};
            }
        fc_norm = (const float *)wslot(by, "fuse.norm");
        t_final = (const float *)wslot(by, "target.final_norm");
        d_final = (const float *)wslot(by, "drafter.final_norm");
        auto fill = [&](const char *pre, const dflash_model_cfg &m, std::vector<LayerW> &v) {
            v.resize(m.n_layers);
            for (int l = 0; l < m.n_layers; ++l) {
                std::string p = std::string(pre) + ".L" + std::to_string(l) + ".";
                LayerW &w = v[l];
                w.attn_norm = (const float *)wslot(by, p + "attn_norm");
                if (m.qk_norm) {
                    w.q_norm = (const float *)wslot(by, p + "q_norm");
                    w.k_norm = (const float *)wslot(by, p + "k_norm");
                }
                w.ffn_norm = (const float *)wslot(by, p + "ffn_norm");
                w.wqkv = wslot(by, p + "wqkv");
                w.wo = wslot(by, p + "wo");
                if (m.n_experts > 0) {
                    w.w_router = wslot(by, p + "w_router");
                    w.we_gate_up = wslot(by, p + "we_gate_up");
                    w.we_down = wslot(by, p + "we_down");
                } else {
                    w.w_gate_up = wslot(by, p + "w_gate_up");
                    w.w_down = wslot(by, p + "w_down");
                }
            }
        };
        fill("target", c.target, tl);
        fill("drafter", c.drafter, dl);
        x = sp<float>(L.x);
        Y = sp<float>(L.Y);
        logits = sp<float>(L.logits);
        plogits = sp<float>(L.plogits);
        if (c.sampling) {
            qlogits = sp<float>(L.qlogits);
            lse_p = sp<float>(L.lse_p);
            lse_q = sp<float>(L.lse_q);
            tok_p = sp<int>(L.tok_p);
            resid = sp<int>(L.resid);
        }
        samp_part = sp<float4>(L.samp_part);
        moe_wt = sp<float>(L.moe_wt);
        moe_part = sp<float>(L.moe_part);
        xn = sp<T>(L.xn);
        dq_in = sp<T>(L.dq_in);
        q = sp<T>(L.q);
        ao = sp<T>(L.ao);
        h = sp<T>(L.h);
        taps_dec = sp<T>(L.taps_dec);
        taps_gather = sp<T>(L.taps_gather);
        taps_pre = sp<T>(L.taps_pre);
        cbuf = sp<T>(L.cbuf);
        tk = sp<T>(L.tk);
        tv = sp<T>(L.tv);
        dk = sp<T>(L.dk);
        dv = sp<T>(L.dv);
        g = sp<int>(L.g);
        drafts = sp<int>(L.drafts);
        accept = sp<int>(L.accept);
        committed = sp<int>(L.committed);
        new_len = sp<int>(L.new_len);
        active = sp<int>(L.active);
        script = sp<int>(L.script);
        out_tok = sp<int>(L.out_tok);
        tokens = sp<int>(L.tokens);
        first_tok = sp<int>(L.first_tok);
        moe_sel = sp<int>(L.moe_sel);
        moe_off = sp<int>(L.moe_off);
        moe_list = sp<int>(L.moe_list);
        st = sp<SeqState>(L.st);
        meta = sp<RowMeta>(L.meta);
        ctx_meta = sp<RowMeta>(L.ctx_meta);
        ctx_meta_pre = sp<RowMeta>(L.ctx_meta_pre);
        rope_t = sp<float2>(L.rope_t);
        rope_d = sp<float2>(L.rope_d);
        stats = sp<DevStats>(L.stats);
        gemm_ws = sp<float>(L.gemm_ws);
        gemm_sem = sp<int>(L.gemm_sem);
        lm_part = sp<float2>(L.lm_part);
        xg_t = sp<T>(L.xg_t);
        moe_xg = sp<T>(L.moe_xg);
        {
            // DFLASH_MOE_STREAM=1: the CUDA-core weight-streaming expert kernels instead
            const char *mv = getenv("DFLASH_MOE_STREAM");
            moe_grouped_on = std::is_same<T, bf16>::value && c.target.n_experts > 0 && !(mv && mv[0] == '1') &&
                             c.target.hidden % 64 == 0 && c.target.expert_ffn % 64 == 0;
        }
        lo_ = L.act_lo;
        xg2 = sp<T>(L.xg2);
        ssq = sp<float>(L.ssq);
        {
            int dev = 0;
            cudaGetDevice(&dev);
            device = dev;
            cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
            const bool bf = std::is_same<T, bf16>::value;
            const int H = c.target.hidden;
            const bool shapes = H % 128 == 0 && num_sms <= 160 && 2 * L.R_dec <= 256;
            // DFLASH_FOLDED_NORM=0 goes back to separate RMSNorm kernels
            // DFLASH_DEP_COUNTERS=1: device completion counters between the kernels of a
            // pass instead of griddepcontrol.wait (same results; measured 0.2 ms per step
            // slower on B200: the fences of every writer cost more than the grid release)
            const char *dv_env = getenv("DFLASH_DEP_COUNTERS");
            dep_on = dv_env && dv_env[0] == '1' && !f8_;  // FP8 / FP4 projections run a quantiser launch first
            const char *fv = getenv("DFLASH_FOLDED_NORM");
            const bool allow = !(fv && fv[0] == '0');
            fold_draft_ok = allow && bf && shapes;
            fold_verify_ok = allow && bf && shapes && c.target.n_experts == 0;
            pv.d_dep = sp<int>(L.dep_v);
            pd.d_dep = sp<int>(L.dep_d);
        }
        att.o_part = sp<float>(L.att_o);
        att.ml_part = sp<float>(L.att_ml);
        att.sem = sp<int>(L.att_sem);
        att.max_parts = L.att_parts;
        att.num_sms = num_sms;
        if constexpr (std::is_same<T, bf16>::value) {
            // DFLASH_ATTN=mma: the cluster-of-kv-heads mma.sync attention instead
            const char *av = getenv("DFLASH_ATTN");
            const bool legacy = av && strcmp(av, "mma") == 0;
            const dflash_model_cfg *ms[2] = {&c.target, &c.drafter};
            T *caches[2][2] = {{tk, tv}, {dk, dv}};
            attn_tma_on = !legacy;
            for (int w = 0; w < 2 && attn_tma_on; ++w) {
                const dflash_model_cfg &m = *ms[w];
                attn_tma_on = attn_tma_supported(m.head_dim, m.n_q_heads / m.n_kv_heads);
                CUtensorMap *dst[2][2] = {{&kv_map[w].k16, &kv_map[w].v16}, {&kv_map[w].k32, &kv_map[w].v32}};
                for (int kt = 0; kt < 2; ++kt)
                    for (int kv = 0; kv < 2 && attn_tma_on; ++kv)
                        attn_tma_on = attn_tma_make_map(dst[kt][kv], (const bf16 *)caches[w][kv], m.head_dim, c.max_len,
                                                        c.max_batch * m.n_kv_heads, m.n_layers, kv_layer_elems(m), lo_,
                                                        kt ? 32 : 16);
            }
            if (!legacy && !attn_tma_on) {
                err = "attention: K/V tensor maps could not be encoded";
                return DFLASH_ECUDA;
            }
        }
        att.n_sem = std::max(L.R_dec, (L.C + 15) / 16) * std::max(c.target.n_kv_heads, c.drafter.n_kv_heads);
        h_len.assign(c.max_batch, 0);
        h_prefilled.assign(c.max_batch, 0);
        // zero the whole state arena once: stale taps / KV never hold NaN bit patterns
        if (cudaMemsetAsync(S, 0, L.state_bytes, s) != cudaSuccess) return fail_cuda("memset state");
        auto rope_table = [&](float2 *tab, const dflash_model_cfg &m) {
            launch_rope_table(tab, c.max_len, m.head_dim, m.rope_theta, m.rope_factor, m.rope_low_freq_factor,
                              m.rope_high_freq_factor, m.rope_original_max_pos, s);
        };
        rope_table(rope_t, c.target);
        rope_table(rope_d, c.drafter);
        if (cudaMallocHost((void **)&pinned, 64) != cudaSuccess) return fail_cuda("pinned host buffer");
        if (cudaEventCreateWithFlags(&ev_a, cudaEventDisableTiming) != cudaSuccess) return fail_cuda("event");
        if (cudaEventCreateWithFlags(&ev_b, cudaEventDisableTiming) != cudaSuccess) return fail_cuda("event");
        if (tc.init(gemm_ws, L.ws_floats, gemm_sem, L.n_sem) != 0) {
            err = "tensor-core GEMM set-up failed: " + tc.err;
            return DFLASH_ECUDA;
        }
        // projection tiling overrides (measurement sweeps); unset = the built-in policy
        auto env_int = [](const char *name) {
            const char *v = getenv(name);
            return v ? atoi(v) : 0;
        };
        tc.tune_splits = env_int("DFLASH_TC_SPLITS");
        tc.tune_smem_kb = env_int("DFLASH_TC_SMEM_KB");
        tc.tune_split_smem_kb = env_int("DFLASH_TC_SPLIT_SMEM_KB");
        tc.tune_ctas_per_sm = env_int("DFLASH_TC_CTAS_PER_SM");
        tc.tune_tm_max = env_int("DFLASH_TC_TM_MAX");
        if (f8_) {
            // every scale byte starts as 1.0 (127): bytes past a projection's K are never NaN
            tc.mx_codes = (uint8_t *)(S + L.mx_codes);
            tc.mx_words = (uint8_t *)(S + L.mx_words);
            tc.mx_mpad = L.mx_mpad;
            tc.mx_kpad = L.mx_kpad;
            if (cudaMemsetAsync(tc.mx_words, 0x7F, (size_t)(L.mx_kpad / 128) * 4 * L.mx_mpad * 4, s) != cudaSuccess)
                return fail_cuda("MX scale buffer");
        }
        tc.set_lm_part(lm_part, (c.target.vocab + 127) / 128 * L.R_dec);
        tc.set_err(&stats->status);
        tc.keep_logits = c.keep_logits;  // plus while sampling (sampling_changed)
        return check("create");
    }

    ~Engine() override {
        for (cudaEvent_t e : ev_pool) cudaEventDestroy(e);
        if (pinned) cudaFreeHost(pinned);
        if (ev_a) cudaEventDestroy(ev_a);
        if (ev_b) cudaEventDestroy(ev_b);
    }

    dflash_status fail_cuda(const char *what) {
        cudaError_t e = cudaGetLastError();
        err = std::string(what) + ": " + cudaGetErrorString(e);
        return DFLASH_ECUDA;
    }

    bool attn_failed = false;  // an attention launch was refused
    bool attn_one_seq = false;  // the attention launches under way are one sequence's prefill chunk
    dflash_status check(const char *what) {
        if (tc.failed) {  // a projection could not be launched (tensor map encoding)
            err = std::string(what) + ": " + tc.err;
            return DFLASH_ECUDA;
        }
        if (attn_failed) {
            err = std::string(what) + ": attention launch failed";
            return DFLASH_ECUDA;
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            err = std::string(what) + ": " + cudaGetErrorString(e);
            return DFLASH_ECUDA;
        }
        return DFLASH_OK;
    }

    dflash_status sync(const char *what) {
        if (cudaEventRecord(ev_a, s) != cudaSuccess) return fail_cuda(what);
        const int tmo = c.timeout_ms > 0 ? c.timeout_ms : 600000;
        auto t0 = std::chrono::steady_clock::now();
        while (true) {
            cudaError_t e = cudaEventQuery(ev_a);
            if (e == cudaSuccess) break;
            if (e != cudaErrorNotReady) {
                err = std::string(what) + ": " + cudaGetErrorString(e);
                return DFLASH_ECUDA;
            }
            auto dt = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0);
            if (dt.count() > tmo) {
                err = std::string(what) + ": stream did not finish within the timeout";
                return DFLASH_ETIMEOUT;
            }
            std::this_thread::sleep_for(std::chrono::microseconds(20));
        }
        return check(what);
    }

    // ---- projections ----
    size_t kv_layer_elems(const dflash_model_cfg &m) const {
        return (size_t)c.max_batch * m.n_kv_heads * c.max_len * m.head_dim;
    }

    cudaEvent_t next_event() {
        if (ev_used == ev_pool.size()) {
            cudaEvent_t e;
            cudaEventCreate(&e);
            ev_pool.push_back(e);
        }
        return ev_pool[ev_used++];
    }

    template <typename F>
    void record(int mode_bit, int c0, int c1, double bytes, F &&launch) {
        if (!(profiling & mode_bit)) {
            launch();
            return;
        }
        ProfRec r{{c0, c1, -1}, bytes, next_event(), next_event()};
        cudaEventRecord(r.a, s);
        launch();
        cudaEventRecord(r.b, s);
        prof.push_back(r);
    }
    template <typename F>
    void timed(int cls, double bytes, F &&launch, int sub = -1) { record(1, cls, sub, bytes, launch); }
    template <typename F>
    void timed_pass(int cls, F &&launch) { record(2, cls, -1, 0.0, launch); }

    // profile class of a projection launch (reporting only)
    int proj_class(int N, int K, int kind) const {
        const int H = c.target.hidden;
        switch (kind) {
            case EPI_QKV: return DFLASH_PROF_QKV;
            case EPI_SWIGLU: return DFLASH_PROF_GATE_UP;
            case EPI_LOGITS: return DFLASH_PROF_LM_HEAD;
            case EPI_NORMOUT: return DFLASH_PROF_FUSE;
            case EPI_RESID: {
                const int qt = c.target.n_q_heads * c.target.head_dim, qd = c.drafter.n_q_heads * c.drafter.head_dim;
                return N == H && (K == qt || K == qd) ? DFLASH_PROF_O : DFLASH_PROF_DOWN;
            }
            default: return K == c.n_taps * H ? DFLASH_PROF_FUSE : DFLASH_PROF_OTHER_PROJ;
        }
    }

    // algorithmic HBM bytes of one projection: the weight matrix once, the
    // activation input (both planes of two-plane activations) and the outputs
    double gemm_bytes(int M, int N, int K, const Epi<T> &e) const {
        const double es = sizeof(T), ea = es * (lo_ ? 2 : 1);
        const int wrows = e.kind == EPI_SWIGLU ? 2 * e.F : N;
        // weights: FP4 half a byte per value + one exponent byte per 32 + the row
        // scales; FP8 one byte per value + the row scales
        double b = f4_ ? (double)wrows * K / 2 + (double)wrows * K / 32 + 4.0 * wrows
                       : f8_ ? (double)wrows * K + 4.0 * wrows : (double)N * K * es;
        b += (double)M * K * ea;
        switch (e.kind) {
            case EPI_QKV: b += (double)M * N * ea; break;
            case EPI_RESID:
                b += (double)M * N * 8 + (double)M * N * ea * e.taps.n + (e.xg ? (double)M * N * ea : 0.0);
                break;
            case EPI_SWIGLU: b += (double)M * e.F * ea; break;
            case EPI_LOGITS: b += (double)((N + 127) / 128) * M * 8; break;
            default: b += (double)M * N * 4; break;
        }
        return b;
    }

    // One projection; returns the CTAs launched (tensor-core path).  dep/done:
    // completion counters of a decode pass (see PassSync), else griddepcontrol.wait.
    // FP8 weights: the row scales of matrix Wt (its base address; rows from row0 on)
    WScales scales_of(const void *Wt, int row0 = 0) const {
        WScales w;
        if (!f8_) return w;
        auto it = wscales.find(Wt);
        if (it != wscales.end()) w.row = it->second + row0;
        if (f4_) {
            auto ib = wbscales.find(Wt);
            if (ib != wbscales.end()) {
                w.blk = ib->second.first;
                w.blk_rows = ib->second.second;
                w.blk_row0 = row0;
            }
        }
        return w;
    }
    // matrix Wt from row row0 on (FP8 codes are one byte per element, FP4 half a byte)
    const void *rows_of(const void *Wt, int row0, int K) const {
        const size_t row_bytes = f4_ ? (size_t)K / 2 : f8_ ? (size_t)K : (size_t)K * sizeof(T);
        return (const char *)Wt + (size_t)row0 * row_bytes;
    }

    int gemm(const T *X, int ldx, int M, const void *Wt, int N, int K, const Epi<T> &e, const int *dep = nullptr,
             int dep_target = 0, int *done = nullptr, WScales ws = WScales()) {
        if (M <= 0) return 0;
        int ctas = 0;
        if (!ws.row) ws = scales_of(Wt);
        timed(DFLASH_PROF_PROJECTION, gemm_bytes(M, N, K, e),
              [&] { ctas = gemm_launch(X, ldx, M, Wt, N, K, e, dep, dep_target, done, ws); }, proj_class(N, K, e.kind));
        return ctas;
    }

    int gemm_launch(const T *X, int ldx, int M, const void *Wt, int N, int K, const Epi<T> &e_in,
                    const int *dep = nullptr, int dep_target = 0, int *done = nullptr, WScales ws = WScales()) {
        Epi<T> e = e_in;
        e.lo = lo_;  // every input and output of the engine's projections lives in the activation span
        if (f8_ && !ws.row) ws = scales_of(Wt);
        if (f8_ && (!ws.row || (f4_ && !ws.blk))) {  // a quantised matrix without its scales: refuse
            tc.failed = true;
            tc.err = "FP8 / FP4 matrix without its scales";
            return 0;
        }
        if (tc.supports(M, N, K))
            return tc.run(X, ldx, M, Wt, N, K, e, s, dep, dep_target, done, ws.row, ws.blk, ws.blk_rows, ws.blk_row0);
        // CUDA-core path (fp32 models): GEMM into fp32 Y, then the epilogue.
        float *Yo = (e.kind == EPI_STORE || e.kind == EPI_LOGITS) ? e.Y : Y;
        const int ldy = (e.kind == EPI_STORE || e.kind == EPI_LOGITS) ? e.ldy : N;
        launch_gemm_simt<T>(X, ldx, M, (const T *)Wt, K, N, K, Yo, ldy, lo_, s);
        switch (e.kind) {
            case EPI_QKV:
                launch_qkv_epilogue<T>(Y, N, e.col0, e.R_blk, M, e.meta, e.ctx_meta, e.nq, e.nkv, e.hd, e.rope,
                                       e.q_out, e.kc, e.vc, e.max_len, lo_, e.qn_g, e.kn_g, e.qk_eps, s);
                break;
            case EPI_RESID:
                launch_residual<T>(e.x, Y, N, N, M, e.taps, lo_, e.meta, s);
                break;
            case EPI_SWIGLU:
                launch_swiglu<T>(Y, N, e.F, M, e.h, e.F, lo_, s);
                break;
            default:
                break;
        }
        return 0;
    }

    // returns the CTAs launched by the tensor-core attention (0 on the CUDA-core path)
    // Query rows per attention tile for blocks of B rows: the attention kernels
    // take at most 16 rows of one sequence per tile, so larger blocks split into
    // equal tiles (the largest divisor of B that is at most 16).
    static int block_tile_rows(int B) {
        for (int t = std::min(B, 16); t > 1; --t)
            if (B % t == 0) return t;
        return 1;
    }

    // attention of layer `layer` of the target (which = 0) or the drafter (1)
    int attention(int which, int layer, const T *qq, const RowMeta *mt, int R, int rows_per_tile, T *out,
                  const AttnSync &sy = AttnSync()) {
        const dflash_model_cfg &m = which ? c.drafter : c.target;
        const T *kc = (which ? dk : tk) + (size_t)layer * kv_layer_elems(m);
        const T *vc = (which ? dv : tv) + (size_t)layer * kv_layer_elems(m);
        const int qd = m.n_q_heads * m.head_dim;
        int ctas = 0;
        timed(DFLASH_PROF_ATTENTION, 0.0, [&] {
            if (attn_tma_on) {
                if constexpr (std::is_same<T, bf16>::value) {
                    AttnTmaArgs a;
                    a.q = (const bf16 *)qq;
                    a.ldq = qd;
                    a.meta = mt;
                    a.R = R;
                    a.rows_per_tile = rows_per_tile;
                    a.nq = m.n_q_heads;
                    a.nkv = m.n_kv_heads;
                    a.max_len = c.max_len;
                    a.n_seq = c.max_batch;
                    a.one_seq = attn_one_seq ? 1 : 0;
                    a.layer = layer;
                    a.scale_log2 = 1.4426950408889634f / sqrtf((float)m.head_dim);
                    a.out = (bf16 *)out;
                    a.ldo = qd;
                    a.lo = lo_;
                    a.err = &stats->status;
                    a.dep_ctr = sy.dep_ctr;
                    a.dep_target = sy.dep_target;
                    a.done_ctr = sy.done_ctr;
                    ctas = launch_attention_tma(kv_map[which], a, m.head_dim, lo_ != 0, num_sms, s);
                    if (ctas < 0) attn_failed = true;
                }
            } else if (attn_mma_supported<T>(m.head_dim))
                ctas = launch_attention_mma<T>(qq, qd, kc, vc, mt, R, rows_per_tile, m.n_q_heads, m.n_kv_heads,
                                               m.head_dim, c.max_len, out, qd, lo_, att, s, sy);
            else
                launch_attention_simt<T>(qq, qd, kc, vc, mt, R, m.n_q_heads, m.n_kv_heads, m.head_dim, c.max_len, out,
                                         qd, s);
        });
        return ctas;
    }

    // QK-norm gains of a layer (fidelity toggle) into a QKV epilogue
    static Epi<T> with_qk_norm(Epi<T> e, const dflash_model_cfg &m, const LayerW &w) {
        if (m.qk_norm) {
            e.qn_g = w.q_norm;
            e.kn_g = w.k_norm;
            e.qk_eps = (float)m.rms_eps;
        }
        return e;
    }

    // one pre-norm decoder layer of the target over R rows in x (meta)
    void target_layer(int l, int R, int rpt, const RowMeta *mt, T *tap_base, int tap_ld) {
        const dflash_model_cfg &m = c.target;
        const LayerW &w = tl[l];
        const int H = m.hidden, hd = m.head_dim, qd = m.n_q_heads * hd, kd = m.n_kv_heads * hd;
        launch_rmsnorm<T>(x, H, w.attn_norm, H, (float)m.rms_eps, xn, H, lo_, R, s);
        Epi<T> e;
        e.kind = EPI_QKV;
        e.R_blk = R;
        e.meta = mt;
        e.nq = m.n_q_heads;
        e.nkv = m.n_kv_heads;
        e.hd = hd;
        e.max_len = c.max_len;
        e.rope = rope_t;
        e.q_out = q;
        e.kc = tk + (size_t)l * kv_layer_elems(m);
        e.vc = tv + (size_t)l * kv_layer_elems(m);
        gemm(xn, H, R, w.wqkv, qd + 2 * kd, H, with_qk_norm(e, m, w));
        attention(0, l, q, mt, R, rpt, ao);
        Epi<T> r;
        r.kind = EPI_RESID;
        r.x = x;
        r.meta = mt;
        gemm(ao, qd, R, w.wo, H, qd, r);
        launch_rmsnorm<T>(x, H, w.ffn_norm, H, (float)m.rms_eps, xn, H, lo_, R, s);
        TapDst<T> taps{};
        taps.base = tap_base;
        taps.ld = tap_ld;
        taps.n = 0;
        if (tap_base)
            for (int i = 0; i < c.n_taps; ++i)
                if (c.tap_layers[i] == l) taps.col[taps.n++] = i * H;
        if (m.n_experts > 0) {
            moe_ffn(l, R, mt, taps);
        } else {
            Epi<T> sw;
            sw.kind = EPI_SWIGLU;
            sw.h = h;
            sw.F = m.ffn;
            gemm(xn, H, R, w.w_gate_up, 2 * m.ffn, H, sw);
            Epi<T> dn;
            dn.kind = EPI_RESID;
            dn.x = x;
            dn.meta = mt;
            dn.taps = taps;
            gemm(h, m.ffn, R, w.w_down, H, m.ffn, dn);
        }
    }

    void moe_ffn(int l, int R, const RowMeta *mt, const TapDst<T> &taps) {
        const dflash_model_cfg &m = c.target;
        const LayerW &w = tl[l];
        const int H = m.hidden, E = m.n_experts, k = m.top_k, Fe = m.expert_ffn;
        Epi<T> e;
        e.kind = EPI_STORE;
        e.Y = Y;
        e.ldy = E;
        gemm(xn, H, R, w.w_router, E, H, e);
        launch_moe_topk(Y, E, R, k, moe_sel, moe_wt, s);
        if constexpr (std::is_same<T, bf16>::value) {
            if (moe_grouped_on && R <= L.R_dec) {
                // decode: each touched expert's gate/up and down as one grouped tcgen05
                // projection over its pairs (rows gathered in expert order)
                int *touched = moe_off + E + 1;
                launch_moe_bucket(moe_sel, R * k, E, moe_off, moe_list, s);
                launch_moe_gather(xn, H, lo_, moe_list, k, R * k, H, moe_xg, s);
                Epi<T> gu;
                gu.kind = EPI_SWIGLU;
                gu.h = h;
                gu.F = Fe;
                gu.lo = lo_;
                timed(DFLASH_PROF_PROJECTION, (double)R * k * H * 2, [&] {
                    tc.run_grouped(moe_xg, H, R * k, (const T *)w.we_gate_up, 2 * Fe, 2 * Fe, H, gu, moe_off, touched,
                                   moe_list, E, R, s);
                }, DFLASH_PROF_OTHER_PROJ);
                Epi<T> dn;
                dn.kind = EPI_STORE;
                dn.Y = moe_part;
                dn.ldy = H;
                dn.lo = lo_;
                timed(DFLASH_PROF_PROJECTION, (double)R * k * Fe * 2, [&] {
                    tc.run_grouped(h, Fe, R * k, (const T *)w.we_down, H, H, Fe, dn, moe_off, touched, moe_list, E, R,
                                   s);
                }, DFLASH_PROF_OTHER_PROJ);
                launch_moe_combine<T>(x, moe_part, moe_wt, H, R, k, taps, lo_, mt, s);
                return;
            }
            if (moe_bucketed_supported(H, Fe, E)) {
                // touched experts only, each expert's weights streamed once per layer
                launch_moe_experts_bucketed(xn, H, lo_, R, k, moe_sel, E, (const bf16 *)w.we_gate_up,
                                            (const bf16 *)w.we_down, H, Fe, moe_off, moe_list, h, lo_, moe_part,
                                            num_sms, &stats->status, s);
                launch_moe_combine<T>(x, moe_part, moe_wt, H, R, k, taps, lo_, mt, s);
                return;
            }
        }
        if (moe_tc_supported<T>()) {
            run_moe_tc<T>(xn, H, R, k, moe_sel, (const T *)w.we_gate_up, (const T *)w.we_down, H, Fe, E, h, moe_part,
                          tc, s);
        } else {
            launch_moe_experts_simt<T>(xn, H, lo_, R, k, moe_sel, (const T *)w.we_gate_up, (const T *)w.we_down, H, Fe,
                                       moe_part, s);
        }
        launch_moe_combine<T>(x, moe_part, moe_wt, H, R, k, taps, lo_, mt, s);
    }

    void drafter_layer(int j, int R, bool with_ctx) {
        const dflash_model_cfg &m = c.drafter;
        const LayerW &w = dl[j];
        const int H = m.hidden, hd = m.head_dim, qd = m.n_q_heads * hd, kd = m.n_kv_heads * hd;
        launch_rmsnorm<T>(x, H, w.attn_norm, H, (float)m.rms_eps, dq_in, H, lo_, R, s);
        Epi<T> e;
        e.kind = EPI_QKV;
        e.R_blk = R;
        e.meta = meta;
        e.ctx_meta = ctx_meta;
        e.nq = m.n_q_heads;
        e.nkv = m.n_kv_heads;
        e.hd = hd;
        e.max_len = c.max_len;
        e.rope = rope_d;
        e.q_out = q;
        e.kc = dk + (size_t)j * kv_layer_elems(m);
        e.vc = dv + (size_t)j * kv_layer_elems(m);
        // block rows and context rows share one pass over Wqkv (K/V injection)
        gemm(dq_in, H, with_ctx ? 2 * R : R, w.wqkv, qd + 2 * kd, H, with_qk_norm(e, m, w));
        attention(1, j, q, meta, R, block_tile_rows(c.block_size), ao);
        Epi<T> r;
        r.kind = EPI_RESID;
        r.x = x;
        r.meta = meta;
        gemm(ao, qd, R, w.wo, H, qd, r);
        launch_rmsnorm<T>(x, H, w.ffn_norm, H, (float)m.rms_eps, xn, H, lo_, R, s);
        Epi<T> sw;
        sw.kind = EPI_SWIGLU;
        sw.h = h;
        sw.F = m.ffn;
        gemm(xn, H, R, w.w_gate_up, 2 * m.ffn, H, sw);
        Epi<T> dn;
        dn.kind = EPI_RESID;
        dn.x = x;
        dn.meta = meta;
        gemm(h, m.ffn, R, w.w_down, H, m.ffn, dn);
    }

    // LM head on normalised rows xin[R][H] -> greedy ids (mode 0: idx[r];
    // mode 1: drafter rows j >= 1 of each block -> idx[i*(B-1)+j-1]), or with
    // smp the temperature-sampled ids of the same rows.
    void head_argmax(const T *xin, int R, float *lg, int mode, int B, int *idx, const SampleRows *smp = nullptr) {
        const int H = c.target.hidden, V = c.target.vocab;
        Epi<T> e;
        e.kind = EPI_LOGITS;
        e.Y = lg;
        e.ldy = V;
        gemm(xin, H, R, lm_head, V, H, e);
        if (smp) launch_sample_rows(*smp, s);
        else if (tc.supports(R, V, H)) launch_lm_argmax(lm_part, (V + 127) / 128, R, mode, B, idx, stats, s);
        else launch_argmax_rows(lg, V, V, R, mode, B, idx, stats, s);
    }

    void lm_head_rows(const float *final_norm, float eps, int R, float *lg, int mode, int B, int *idx,
                      const SampleRows *smp = nullptr) {
        const int H = c.target.hidden;
        launch_rmsnorm<T>(x, H, final_norm, H, eps, xn, H, lo_, R, s);
        head_argmax(xn, R, lg, mode, B, idx, smp);
    }

    // ---- temperature sampling ----
    bool sampling_on() const { return temperature > 0.f; }
    // the sampling kernels read the fp32 logits rows the LM heads store; greedy
    // passes store them only for dflash_debug_logits
    void sampling_changed() override { tc.keep_logits = c.keep_logits || sampling_on(); }
    float *draft_logits() { return c.sampling ? qlogits : logits; }

    // rows [R] of logits lg (block B, row k of sequence i drawn at st.len + k + pos_off)
    SampleRows sample_desc(const float *lg, int R, int B, int mode, uint32_t purpose, int pos_off, int *tok,
                           float *lse) {
        SampleRows a;
        a.logits = lg;
        a.ldl = a.V = c.target.vocab;
        a.R = R;
        a.B = B;
        a.mode = mode;
        a.inv_T = 1.f / temperature;
        a.key = sample_key(seed);
        a.purpose = purpose;
        a.pos_off = pos_off;
        a.st = st;
        a.active = active;
        a.part = samp_part;
        a.lse = lse;
        a.tok = tok;
        a.stats = stats;
        return a;
    }

    // after the verify head's draws (tok_p, lse_p): residual draws and the acceptance
    void accept_sampled(int nseq) {
        const int B = c.block_size, V = c.target.vocab;
        if (B > 1) {
            ResidualRows r;
            r.plog = logits;
            r.qlog = qlogits;
            r.ldl = r.V = V;
            r.B = B;
            r.rows = nseq * (B - 1);
            r.inv_T = 1.f / temperature;
            r.key = sample_key(seed);
            r.lse_p = lse_p;
            r.lse_q = lse_q;
            r.st = st;
            r.active = active;
            r.part = reinterpret_cast<float2 *>(samp_part);
            r.resid = resid;
            launch_residual_rows(r, s);
        }
        AcceptSample a;
        a.st = st;
        a.active = active;
        a.nseq = nseq;
        a.B = B;
        a.drafts = drafts;
        a.plog = logits;
        a.qlog = qlogits;
        a.ldl = V;
        a.lse_p = lse_p;
        a.lse_q = lse_q;
        a.inv_T = 1.f / temperature;
        a.key = sample_key(seed);
        a.resid = resid;
        a.tok_p = tok_p;
        a.accept = accept;
        a.committed = committed;
        a.new_len = new_len;
        a.out_tok = out_tok;
        a.out_ld = c.max_len;
        a.stats = stats;
        launch_accept_sample(a, s);
    }

    // ---- folded-norm decode passes (bf16) ----
    // Append one projection to a pass program.
    void prog_add(PassProgram &pg, int kind, const void *W, int N, int K, const T *X, int ldx, int M, const Epi<T> &e) {
        if constexpr (std::is_same<T, bf16>::value) {
            PassOp op;
            op.kind = kind;
            op.e = e;
            op.e.lo = lo_;
            pg.ops.push_back(op);
            pg.hops.push_back(HostOp{W, N, K, X, ldx, M});
        }
    }

    void finish_program(PassProgram &pg) {
        cudaMemsetAsync(pg.d_dep, 0, sizeof(int) * 2 * pg.ops.size(), s);
        pg.dep_run = 0;
        pg.dep_ctas.assign(2 * pg.ops.size(), 0);
        pg.dep_prev = -1;
    }

    Epi<T> epi_norm_in(Epi<T> e, float eps, int H) {
        e.rs_ssq = ssq;
        e.rs_tiles = H / 128;
        e.rs_ld = L.ssq_ld;
        e.rs_inv_n = 1.0f / (float)H;
        e.rs_eps = eps;
        return e;
    }

    Epi<T> epi_norm_out(Epi<T> e, T *xg, const float *g, float *ssq_out) {
        e.xg = xg;
        e.xg_ld = c.target.hidden;
        e.g_next = g;
        e.ssq_out = ssq_out;
        e.ssq_ld = L.ssq_ld;
        return e;
    }

    // verify: QKV(0) | per layer O, gate/up, down, QKV(l+1) or LM head
    void build_verify_program(int nseq) {
        const dflash_model_cfg &m = c.target;
        const int B = c.block_size, R = nseq * B, H = m.hidden, hd = m.head_dim;
        const int qd = m.n_q_heads * hd, kd = m.n_kv_heads * hd, TK = c.n_taps * H;
        PassProgram &pg = pv;
        pg.ops.clear();
        pg.hops.clear();
        pg.key = nseq;
        auto qkv = [&](int l) {
            Epi<T> e;
            e.kind = EPI_QKV;
            e.R_blk = R;
            e.meta = meta;
            e.nq = m.n_q_heads;
            e.nkv = m.n_kv_heads;
            e.hd = hd;
            e.max_len = c.max_len;
            e.rope = rope_t;
            e.q_out = q;
            e.kc = tk + (size_t)l * kv_layer_elems(m);
            e.vc = tv + (size_t)l * kv_layer_elems(m);
            prog_add(pg, EPI_QKV, tl[l].wqkv, qd + 2 * kd, H, xg_t, H, R,
                     epi_norm_in(with_qk_norm(e, m, tl[l]), (float)m.rms_eps, H));
        };
        qkv(0);
        for (int l = 0; l < m.n_layers; ++l) {
            Epi<T> o;
            o.kind = EPI_RESID;
            o.x = x;
            o.meta = meta;
            prog_add(pg, EPI_RESID, tl[l].wo, H, qd, ao, qd, R, epi_norm_out(o, xg2, tl[l].ffn_norm, ssq));
            Epi<T> gu;
            gu.kind = EPI_SWIGLU;
            gu.h = h;
            gu.F = m.ffn;
            prog_add(pg, EPI_SWIGLU, tl[l].w_gate_up, 2 * m.ffn, H, xg2, H, R, epi_norm_in(gu, (float)m.rms_eps, H));
            Epi<T> dn;
            dn.kind = EPI_RESID;
            dn.x = x;
            dn.meta = meta;
            TapDst<T> taps{};
            taps.base = taps_dec;
            taps.ld = TK;
            for (int i = 0; i < c.n_taps; ++i)
                if (c.tap_layers[i] == l) taps.col[taps.n++] = i * H;
            dn.taps = taps;
            const float *gn = l + 1 < m.n_layers ? tl[l + 1].attn_norm : t_final;
            prog_add(pg, EPI_RESID, tl[l].w_down, H, m.ffn, h, m.ffn, R, epi_norm_out(dn, xg_t, gn, ssq));
            if (l + 1 < m.n_layers) {
                qkv(l + 1);
            } else {
                Epi<T> lg;
                lg.kind = EPI_LOGITS;
                lg.Y = logits;
                lg.ldy = m.vocab;
                prog_add(pg, EPI_LOGITS, lm_head, m.vocab, H, xg_t, H, R, epi_norm_in(lg, (float)m.rms_eps, H));
            }
        }
        finish_program(pg);
    }

    // draft: fuse (context rows) + QKV(0) | per layer O, gate/up, down, QKV(j+1) or LM head
    void build_draft_program(int nseq) {
        const dflash_model_cfg &m = c.drafter;
        const int B = c.block_size, R = nseq * B, H = m.hidden, hd = m.head_dim;
        const int qd = m.n_q_heads * hd, kd = m.n_kv_heads * hd, TK = c.n_taps * c.target.hidden;
        PassProgram &pg = pd;
        pg.ops.clear();
        pg.hops.clear();
        pg.key = nseq;
        Epi<T> f;
        f.kind = EPI_NORMOUT;
        prog_add(pg, EPI_NORMOUT, w_fc, H, TK, taps_dec, TK, R, epi_norm_out(f, dq_in + (size_t)R * H, fc_norm, ssq + R));
        auto qkv = [&](int j) {
            Epi<T> e;
            e.kind = EPI_QKV;
            e.R_blk = R;
            e.meta = meta;
            e.ctx_meta = ctx_meta;
            e.nq = m.n_q_heads;
            e.nkv = m.n_kv_heads;
            e.hd = hd;
            e.max_len = c.max_len;
            e.rope = rope_d;
            e.q_out = q;
            e.kc = dk + (size_t)j * kv_layer_elems(m);
            e.vc = dv + (size_t)j * kv_layer_elems(m);
            prog_add(pg, EPI_QKV, dl[j].wqkv, qd + 2 * kd, H, dq_in, H, 2 * R,
                     epi_norm_in(with_qk_norm(e, m, dl[j]), (float)m.rms_eps, H));
        };
        qkv(0);
        for (int j = 0; j < m.n_layers; ++j) {
            Epi<T> o;
            o.kind = EPI_RESID;
            o.x = x;
            o.meta = meta;
            prog_add(pg, EPI_RESID, dl[j].wo, H, qd, ao, qd, R, epi_norm_out(o, xg2, dl[j].ffn_norm, ssq));
            Epi<T> gu;
            gu.kind = EPI_SWIGLU;
            gu.h = h;
            gu.F = m.ffn;
            prog_add(pg, EPI_SWIGLU, dl[j].w_gate_up, 2 * m.ffn, H, xg2, H, R, epi_norm_in(gu, (float)m.rms_eps, H));
            Epi<T> dn;
            dn.kind = EPI_RESID;
            dn.x = x;
            dn.meta = meta;
            if (j + 1 < m.n_layers) {
                prog_add(pg, EPI_RESID, dl[j].w_down, H, m.ffn, h, m.ffn, R, epi_norm_out(dn, dq_in, dl[j + 1].attn_norm, ssq));
                qkv(j + 1);
            } else {
                prog_add(pg, EPI_RESID, dl[j].w_down, H, m.ffn, h, m.ffn, R, epi_norm_out(dn, xg_t, d_final, ssq));
                Epi<T> lg;
                lg.kind = EPI_LOGITS;
                lg.Y = draft_logits();
                lg.ldy = c.target.vocab;
                prog_add(pg, EPI_LOGITS, lm_head, c.target.vocab, H, xg_t, H, R, epi_norm_in(lg, (float)m.rms_eps, H));
            }
        }
        finish_program(pg);
    }

    // ops [b, e) of a program, one projection kernel each
    void run_ops(PassProgram &pg, int b, int e) {
        if constexpr (std::is_same<T, bf16>::value) {
            for (int i = b; i < e; ++i) {
                const HostOp &h = pg.hops[i];
                int tgt = 0;
                const int *dep = pass_dep(pg, tgt);
                const int k = gemm((const T *)h.X, h.ldx, h.M, h.W, h.N, h.K, pg.ops[i].e, dep, tgt,
                                   dep_on ? pg.d_dep + i : nullptr);
                pass_done(pg, i, k);
            }
        }
    }

    // Completion counters of a decode pass run one kernel per projection: each
    // projection and attention launch waits until every CTA of the launch before
    // it has signalled (instead of waiting for that grid to exit and flush), which
    // lets it start about as soon as the last epilogue store is visible.
    void pass_begin(PassProgram &pg) {
        pg.dep_run += 1;
        pg.dep_prev = -1;  // the first launch of a pass waits with griddepcontrol.wait
    }
    const int *pass_dep(PassProgram &pg, int &target) {
        if (!dep_on || pg.dep_prev < 0) {
            target = 0;
            return nullptr;
        }
        target = (int)pg.dep_run * pg.dep_ctas[pg.dep_prev];
        return pg.d_dep + pg.dep_prev;
    }
    void pass_done(PassProgram &pg, int idx, int ctas) {
        if (!dep_on) return;
        pg.dep_ctas[idx] = ctas;
        pg.dep_prev = ctas > 0 ? idx : -1;  // a launch that signals nothing cannot be waited on
    }
    AttnSync pass_attn_sync(PassProgram &pg, int layer, int &idx) {
        AttnSync sy;
        idx = (int)pg.ops.size() + layer;
        if (!dep_on) return sy;
        sy.dep_ctr = pass_dep(pg, sy.dep_target);
        sy.done_ctr = pg.d_dep + idx;
        sy.err = &stats->status;
        return sy;
    }

    void enqueue_verify_folded(int nseq) {
        const dflash_model_cfg &t = c.target;
        const int B = c.block_size, R = nseq * B, H = t.hidden;
        if (pv.key != nseq) build_verify_program(nseq);
        pass_begin(pv);
        launch_embed_norm<T>(embed, H, st, active, nseq, B, 0, drafts, c.mask_token_id, x, meta, nullptr, tl[0].attn_norm,
                             xg_t, H, lo_, ssq, L.ssq_ld, s);
        run_ops(pv, 0, 1);
        for (int l = 0; l < t.n_layers; ++l) {
            int ai;
            const AttnSync sy = pass_attn_sync(pv, l, ai);
            const int k = attention(0, l, q, meta, R, block_tile_rows(B), ao, sy);
            pass_done(pv, ai, k);
            run_ops(pv, 1 + 4 * l, 5 + 4 * l);
        }
        if (sampling_on()) {
            launch_sample_rows(sample_desc(logits, R, B, 0, SP_TARGET, 1, tok_p, lse_p), s);
            accept_sampled(nseq);
        } else {
            launch_lm_argmax(lm_part, (t.vocab + 127) / 128, R, 0, B, g, stats, s);
            launch_accept(st, active, nseq, B, drafts, g, accept, committed, new_len, out_tok, c.max_len, stats, s);
        }
        fold_used[1] = true;
    }

    void enqueue_draft_folded(int nseq) {
        const dflash_model_cfg &d = c.drafter;
        const int B = c.block_size, R = nseq * B, H = d.hidden;
        if (pd.key != nseq) build_draft_program(nseq);
        pass_begin(pd);
        launch_embed_norm<T>(embed, H, st, active, nseq, B, 1, nullptr, c.mask_token_id, x, meta, ctx_meta, dl[0].attn_norm,
                             dq_in, H, lo_, ssq, L.ssq_ld, s);
        run_ops(pd, 0, 2);
        for (int j = 0; j < d.n_layers; ++j) {
            int ai;
            const AttnSync sy = pass_attn_sync(pd, j, ai);
            const int k = attention(1, j, q, meta, R, block_tile_rows(B), ao, sy);
            pass_done(pd, ai, k);
            run_ops(pd, 2 + 4 * j, 6 + 4 * j);
        }
        if (B > 1) {
            if (sampling_on())
                launch_sample_rows(sample_desc(qlogits, R, B, 1, SP_DRAFT, 0, drafts, lse_q), s);
            else
                launch_lm_argmax(lm_part, (c.target.vocab + 127) / 128, R, 1, B, drafts, stats, s);
        }
        if (draft_mode == DFLASH_DRAFT_SCRIPT)
            launch_script_drafts(st, active, nseq, B, tau, c.target.vocab, script, c.max_len, drafts, s);
        fold_used[0] = true;
    }

    // ---- steps ----
    void enqueue_prefill(int seq, int n, int max_new) {
        const dflash_model_cfg &t = c.target, &d = c.drafter;
        const int H = t.hidden, TK = c.n_taps * H;
        const int qd = d.n_q_heads * d.head_dim, kd = d.n_kv_heads * d.head_dim;
        for (int c0 = 0; c0 < n; c0 += L.C) {
            const int R = std::min(L.C, n - c0);
            launch_embed_tokens<T>(embed, H, tokens + c0, R, seq, c0, x, meta, s);
            attn_one_seq = true;
            for (int l = 0; l < t.n_layers; ++l) target_layer(l, R, 16, meta, taps_pre, TK);
            attn_one_seq = false;
            if (c0 + R == n) {
                // first token from the last prompt row: greedy, or the target's draw at position n
                launch_rmsnorm<T>(x + (size_t)(R - 1) * H, H, t_final, H, (float)t.rms_eps, xn, H, lo_, 1, s);
                if (sampling_on()) {
                    SampleRows a = sample_desc(plogits, 1, 1, 0, SP_TARGET, 0, first_tok, nullptr);
                    a.fixed_pos = n;
                    a.fixed_slot = seq;
                    head_argmax(xn, 1, plogits, 0, 1, first_tok, &a);
                } else {
                    head_argmax(xn, 1, plogits, 0, 1, first_tok);
                }
            }
            // context vectors of the prompt rows -> drafter context K/V
            Epi<T> f;
            f.kind = EPI_STORE;
            f.Y = Y;
            f.ldy = H;
            gemm(taps_pre, TK, R, w_fc, H, TK, f);
            launch_rmsnorm<T>(Y, H, fc_norm, H, (float)d.rms_eps, cbuf, H, lo_, R, s);
            launch_ctx_meta_prefill(ctx_meta_pre, R, seq, c0, s);
            for (int j = 0; j < d.n_layers; ++j) {
                Epi<T> e;
                e.kind = EPI_QKV;
                e.col0 = qd;
                e.R_blk = 0;
                e.ctx_meta = ctx_meta_pre;
                e.nq = d.n_q_heads;
                e.nkv = d.n_kv_heads;
                e.hd = d.head_dim;
                e.max_len = c.max_len;
                e.rope = rope_d;
                e.kc = dk + (size_t)j * kv_layer_elems(d);
                e.vc = dv + (size_t)j * kv_layer_elems(d);
                // rows qd .. qd + 2kd of Wqkv are [Wk; Wv]
                gemm(cbuf, H, R, rows_of(dl[j].wqkv, qd, H), 2 * kd, H, with_qk_norm(e, d, dl[j]), nullptr, 0, nullptr,
                     scales_of(dl[j].wqkv, qd));
            }
        }
        launch_prefill_finish(st, seq, n, first_tok, out_tok, c.max_len, max_new, s);
    }

    void enqueue_draft(int nseq, bool contiguous) {
        if (fold_draft_ok && contiguous) {
            if (pd.key != nseq) build_draft_program(nseq);
            enqueue_draft_folded(nseq);
            return;
        }
        fold_used[0] = false;
        const dflash_model_cfg &t = c.target, &d = c.drafter;
        const int B = c.block_size, R = nseq * B, H = t.hidden, TK = c.n_taps * H;
        launch_embed_block<T>(embed, H, st, active, nseq, B, 1, nullptr, c.mask_token_id, x, meta, ctx_meta, s);
        // fuse pending taps -> context vectors (rows R..2R-1 of the drafter QKV input)
        const T *tin = taps_dec;
        if (!contiguous) {
            launch_gather_rows(taps_dec, taps_gather, (size_t)TK * sizeof(T), active, nseq, B, s);
            if (lo_) launch_gather_rows(taps_dec + lo_, taps_gather + lo_, (size_t)TK * sizeof(T), active, nseq, B, s);
            tin = taps_gather;
        }
        Epi<T> f;
        f.kind = EPI_STORE;
        f.Y = Y;
        f.ldy = H;
        gemm(tin, TK, R, w_fc, H, TK, f);
        launch_rmsnorm<T>(Y, H, fc_norm, H, (float)d.rms_eps, dq_in + (size_t)R * H, H, lo_, R, s);
        for (int j = 0; j < d.n_layers; ++j) drafter_layer(j, R, true);
        if (B > 1) {
            if (sampling_on()) {
                const SampleRows a = sample_desc(qlogits, R, B, 1, SP_DRAFT, 0, drafts, lse_q);
                lm_head_rows(d_final, (float)d.rms_eps, R, qlogits, 1, B, drafts, &a);
            } else {
                lm_head_rows(d_final, (float)d.rms_eps, R, draft_logits(), 1, B, drafts);
            }
        }
        if (draft_mode == DFLASH_DRAFT_SCRIPT)
            launch_script_drafts(st, active, nseq, B, tau, t.vocab, script, c.max_len, drafts, s);
    }

    void enqueue_verify(int nseq) {
        if (fold_verify_ok) {
            if (pv.key != nseq) build_verify_program(nseq);
            enqueue_verify_folded(nseq);
            return;
        }
        fold_used[1] = false;
        const dflash_model_cfg &t = c.target;
        const int B = c.block_size, R = nseq * B, H = t.hidden, TK = c.n_taps * H;
        launch_embed_block<T>(embed, H, st, active, nseq, B, 0, drafts, c.mask_token_id, x, meta, nullptr, s);
        for (int l = 0; l < t.n_layers; ++l) target_layer(l, R, block_tile_rows(B), meta, taps_dec, TK);
        if (sampling_on()) {
            const SampleRows a = sample_desc(logits, R, B, 0, SP_TARGET, 1, tok_p, lse_p);
            lm_head_rows(t_final, (float)t.rms_eps, R, logits, 0, B, tok_p, &a);
            accept_sampled(nseq);
        } else {
            lm_head_rows(t_final, (float)t.rms_eps, R, logits, 0, B, g);
            launch_accept(st, active, nseq, B, drafts, g, accept, committed, new_len, out_tok, c.max_len, stats, s);
        }
    }

    void enqueue_ar_step(int nseq) {
        const dflash_model_cfg &t = c.target;
        const int H = t.hidden;
        launch_embed_block<T>(embed, H, st, active, nseq, 1, 0, drafts, c.mask_token_id, x, meta, nullptr, s);
        for (int l = 0; l < t.n_layers; ++l) target_layer(l, nseq, 1, meta, nullptr, 0);
        if (sampling_on()) {
            const SampleRows a = sample_desc(logits, nseq, 1, 0, SP_TARGET, 1, g, nullptr);
            lm_head_rows(t_final, (float)t.rms_eps, nseq, logits, 0, 1, g, &a);
        } else {
            lm_head_rows(t_final, (float)t.rms_eps, nseq, logits, 0, 1, g);
        }
        launch_ar_step(st, active, nseq, g, out_tok, c.max_len, stats, s);
    }

    // ---- API ----
    dflash_status refresh_lens() {
        if (!lens_stale) return DFLASH_OK;
        dflash_status r = sync("lengths");
        if (r) return r;
        std::vector<SeqState> hs(c.max_batch);
        if (cudaMemcpy(hs.data(), st, sizeof(SeqState) * c.max_batch, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("state copy");
        for (int i = 0; i < c.max_batch; ++i)
            if (h_prefilled[i]) h_len[i] = hs[i].len;
        lens_stale = false;
        return DFLASH_OK;
    }

    dflash_status check_seqs(const int32_t *seqs, int n) {
        if (!seqs || n < 1 || n > c.max_batch) { err = "seqs must hold 1..max_batch slots"; return DFLASH_EINVAL; }
        dflash_status rr = refresh_lens();
        if (rr) return rr;
        std::vector<char> seen(c.max_batch, 0);
        for (int i = 0; i < n; ++i) {
            if (seqs[i] < 0 || seqs[i] >= c.max_batch || seen[seqs[i]]) { err = "bad or repeated slot"; return DFLASH_EINVAL; }
            seen[seqs[i]] = 1;
            if (!h_prefilled[seqs[i]]) { err = "slot not prefilled"; return DFLASH_ESTATE; }
            if (h_len[seqs[i]] + c.block_size > c.max_len) { err = "sequence would exceed max_len"; return DFLASH_ECAPACITY; }
        }
        return DFLASH_OK;
    }

    dflash_status prefill(int seq, const int32_t *prompt, int n, int max_new, int32_t *first) override {
        if (seq < 0 || seq >= c.max_batch || !prompt || n < 1) { err = "bad prefill arguments"; return DFLASH_EINVAL; }
        if (n + c.block_size > c.max_len) { err = "prompt + block exceeds max_len"; return DFLASH_ECAPACITY; }
        for (int i = 0; i < n; ++i)
            if (prompt[i] < 0 || prompt[i] >= c.target.vocab) { err = "prompt id out of vocab"; return DFLASH_EINVAL; }
        last_pass = PASS_NONE;
        if (cudaMemcpyAsync(tokens, prompt, sizeof(int32_t) * n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return fail_cuda("prompt copy");
        enqueue_prefill(seq, n, max_new);
        dflash_status r = check("prefill launch");
        if (r) return r;
        last_pass = PASS_PREFILL;
        h_len[seq] = n;
        h_prefilled[seq] = 1;
        last_draft.clear();
        last_logits_rows[2] = 1;
        if (first) {
            if ((r = sync("prefill"))) return r;
            if ((r = numeric_status())) return r;
            if (cudaMemcpy(first, first_tok, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return fail_cuda("first token");
        }
        return DFLASH_OK;
    }

    dflash_status set_active(const int32_t *seqs, int n) {
        if (cudaMemcpyAsync(active, seqs, sizeof(int32_t) * n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return fail_cuda("active copy");
        return DFLASH_OK;
    }

    static bool is_iota(const int32_t *seqs, int n) {
        for (int i = 0; i < n; ++i) if (seqs[i] != i) return false;
        return true;
    }

    dflash_status draft(const int32_t *seqs, int n, int32_t *out, bool) override {
        dflash_status r = check_seqs(seqs, n);
        if (r) return r;
        if ((r = set_active(seqs, n))) return r;
        last_pass = PASS_NONE;
        timed_pass(DFLASH_PROF_DRAFT_PASS, [&] { enqueue_draft(n, is_iota(seqs, n)); });
        if ((r = check("draft launch"))) return r;
        last_pass = PASS_DRAFT;
        last_draft.assign(seqs, seqs + n);
        last_logits_rows[0] = n * c.block_size;
        if (out && c.block_size > 1) {
            if ((r = sync("draft"))) return r;
            if ((r = numeric_status())) return r;
            if (cudaMemcpy(out, drafts, sizeof(int32_t) * n * (c.block_size - 1), cudaMemcpyDeviceToHost) != cudaSuccess)
                return fail_cuda("drafts copy");
        }
        return DFLASH_OK;
    }

    dflash_status verify(const int32_t *seqs, int n, const int32_t *dr, int32_t *acc, int32_t *com,
                         int32_t *nl) override {
        dflash_status r = check_seqs(seqs, n);
        if (r) return r;
        if ((int)last_draft.size() != n || !std::equal(last_draft.begin(), last_draft.end(), seqs)) {
            err = "verify_commit must follow dflash_draft_block on the same sequences";
            return DFLASH_ESTATE;
        }
        const int B = c.block_size;
        if (dr) {
            for (int i = 0; i < n * (B - 1); ++i)
                if (dr[i] < 0 || dr[i] >= c.target.vocab) { err = "draft id out of vocab"; return DFLASH_EINVAL; }
            if (B > 1 && cudaMemcpyAsync(drafts, dr, sizeof(int32_t) * n * (B - 1), cudaMemcpyHostToDevice, s) != cudaSuccess)
                return fail_cuda("drafts copy");
        }
        last_pass = PASS_NONE;
        timed_pass(DFLASH_PROF_VERIFY_PASS, [&] { enqueue_verify(n); });
        if ((r = check("verify launch"))) return r;
        last_pass = PASS_VERIFY;
        last_draft.clear();
        last_logits_rows[1] = n * B;
        if ((r = sync("verify"))) return r;
        std::vector<int32_t> lens(n);
        if (cudaMemcpy(lens.data(), new_len, sizeof(int32_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("new_len copy");
        for (int i = 0; i < n; ++i) h_len[seqs[i]] = lens[i];
        if ((r = numeric_status())) return r;
        if (nl) std::copy(lens.begin(), lens.end(), nl);
        if (acc && cudaMemcpy(acc, accept, sizeof(int32_t) * n, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("accept copy");
        if (com && cudaMemcpy(com, committed, sizeof(int32_t) * n * B, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("committed copy");
        return DFLASH_OK;
    }

    // The device status word (stream already synchronised): bit 0 a non-finite
    // logit reached an argmax, bits 2-5 a bounded device wait expired.  Sticky
    // until dflash_reset_stats or the next generation.
    static dflash_status status_code(int st, std::string &err) {
        if (st & 1) { err = "non-finite logits reached an argmax"; return DFLASH_ENUMERIC; }
        if (st & (4 | 8 | 16 | 32)) {
            // which waits gave up: 4 an mbarrier, 8 a completion counter, 16 an
            // attention split counter, 32 an attention input wait
            char buf[96];
            snprintf(buf, sizeof buf, "a bounded device wait expired (status bits 0x%x)", st & 60);
            err = buf;
            return DFLASH_ETIMEOUT;
        }
        return DFLASH_OK;
    }
    dflash_status numeric_status() {
        int32_t st = 0;
        if (cudaMemcpy(&st, &stats->status, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("status copy");
        return status_code(st, err);
    }

    dflash_status start_run(const int32_t *const *prompts, const int32_t *lens, int n, int max_new) {
        if (!prompts || !lens || n < 1 || n > c.max_batch || max_new < 1) { err = "bad generate arguments"; return DFLASH_EINVAL; }
        for (int i = 0; i < n; ++i) {
            if (!prompts[i] || lens[i] < 1) { err = "empty prompt"; return DFLASH_EINVAL; }
            if ((int64_t)lens[i] + max_new + c.block_size > c.max_len) { err = "prompt + max_new + block exceeds max_len"; return DFLASH_ECAPACITY; }
        }
        if (cudaMemsetAsync(stats, 0, sizeof(DevStats), s) != cudaSuccess) return fail_cuda("stats reset");
        for (int i = 0; i < n; ++i) {
            dflash_status r = prefill(i, prompts[i], lens[i], max_new, nullptr);
            if (r) return r;
        }
        std::vector<int32_t> iota(n);
        for (int i = 0; i < n; ++i) iota[i] = i;
        return set_active(iota.data(), n);
    }

    // Run iterations until every sequence is done; the done counter of
    // iteration k is read while iteration k+1 is already queued.
    template <typename F>
    dflash_status run_loop(int n, int max_iters, F &&step, int64_t *iters_out) {
        int64_t it = 0;
        bool pending = false;
        while (it < max_iters) {
            step();
            ++it;
            if (cudaMemcpyAsync(pinned + (it & 1), &stats->n_done, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
                return fail_cuda("done counter");
            cudaEvent_t ev = (it & 1) ? ev_a : ev_b;
            if (cudaEventRecord(ev, s) != cudaSuccess) return fail_cuda("event");
            if (pending) {
                cudaEvent_t prev = (it & 1) ? ev_b : ev_a;
                const int tmo = c.timeout_ms > 0 ? c.timeout_ms : 600000;
                auto t0 = std::chrono::steady_clock::now();
                while (true) {
                    cudaError_t e = cudaEventQuery(prev);
                    if (e == cudaSuccess) break;
                    if (e != cudaErrorNotReady) { err = cudaGetErrorString(e); return DFLASH_ECUDA; }
                    if (std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count() > tmo) {
                        err = "decode iteration did not finish within the timeout";
                        return DFLASH_ETIMEOUT;
                    }
                    std::this_thread::yield();
                }
                if (pinned[(it - 1) & 1] >= n) break;
            }
            pending = true;
        }
        dflash_status r = sync("decode");
        if (r) return r;
        if (iters_out) *iters_out = it;
        return check("decode loop");
    }

    // CUDA events destroyed on every return path
    struct ScopedEvents {
        cudaEvent_t e[3] = {nullptr, nullptr, nullptr};
        ScopedEvents() {
            for (auto &x : e) cudaEventCreate(&x);
        }
        ~ScopedEvents() {
            for (auto &x : e)
                if (x) cudaEventDestroy(x);
        }
    };

    dflash_status generate(const int32_t *const *prompts, const int32_t *lens, int n, int max_new, int32_t *out,
                           dflash_stats *ost) override {
        ScopedEvents ev;
        OtherPass mark{last_pass};
        cudaEvent_t t0 = ev.e[0], t1 = ev.e[1], t2 = ev.e[2];
        cudaEventRecord(t0, s);
        dflash_status r = start_run(prompts, lens, n, max_new);
        if (r) return r;
        cudaEventRecord(t1, s);
        const bool contiguous = true;
        if (max_new > 1) {
            r = run_loop(n, max_new + 2, [&] { enqueue_draft(n, contiguous); enqueue_verify(n); }, nullptr);
            if (r) return r;
        }
        cudaEventRecord(t2, s);
        if ((r = sync("generate"))) return r;
        for (int i = 0; i < n; ++i)
            if (cudaMemcpy(out + (size_t)i * max_new, out_tok + (size_t)i * c.max_len, sizeof(int32_t) * max_new,
                           cudaMemcpyDeviceToHost) != cudaSuccess)
                return fail_cuda("output copy");
        DevStats hs;
        if (cudaMemcpy(&hs, stats, sizeof hs, cudaMemcpyDeviceToHost) != cudaSuccess) return fail_cuda("stats");
        for (int i = 0; i < n; ++i) h_len[i] = 0;
        if (ost) {
            memset(ost, 0, sizeof *ost);
            ost->iterations = (int64_t)hs.iterations;
            ost->tokens = (int64_t)hs.tokens;
            for (int i = 0; i < DFLASH_MAX_BLOCK; ++i) ost->accept_hist[i] = (int64_t)hs.hist[i];
            ost->mean_tau = hs.iterations ? (double)hs.tokens / (double)hs.iterations : 0.0;
            float a = 0, b = 0;
            cudaEventElapsedTime(&a, t0, t1);
            cudaEventElapsedTime(&b, t1, t2);
            ost->ms_prefill = a;
            ost->ms_decode = b;
            ost->kernel_launches = launch_count();
        }
        // generation leaves the slots in a finished state: refuse draft/verify on them
        for (int i = 0; i < n; ++i) h_prefilled[i] = 0;
        if ((r = status_code(hs.status, err))) return r;
        return check("generate");
    }

    dflash_status generate_ar(const int32_t *const *prompts, const int32_t *lens, int n, int max_new, int32_t *out,
                              double *ms) override {
        ScopedEvents ev;
        OtherPass mark{last_pass};
        cudaEvent_t t1 = ev.e[0], t2 = ev.e[1];
        dflash_status r = start_run(prompts, lens, n, max_new);
        if (r) return r;
        cudaEventRecord(t1, s);
        if (max_new > 1) {
            r = run_loop(n, max_new + 1, [&] { enqueue_ar_step(n); }, nullptr);
            if (r) return r;
        }
        cudaEventRecord(t2, s);
        if ((r = sync("generate_ar"))) return r;
        for (int i = 0; i < n; ++i)
            if (cudaMemcpy(out + (size_t)i * max_new, out_tok + (size_t)i * c.max_len, sizeof(int32_t) * max_new,
                           cudaMemcpyDeviceToHost) != cudaSuccess)
                return fail_cuda("output copy");
        if (ms) {
            float b = 0;
            cudaEventElapsedTime(&b, t1, t2);
            *ms = b;
        }
        for (int i = 0; i < n; ++i) h_prefilled[i] = 0;
        return numeric_status();
    }

    dflash_status debug_logits(int which, float *out, int64_t cap, int64_t *rows) override {
        if (!c.keep_logits) { err = "context created without keep_logits"; return DFLASH_ESTATE; }
        if (which < 0 || which > 2 || !out) { err = "bad debug_logits arguments"; return DFLASH_EINVAL; }
        const int64_t V = c.target.vocab;
        const int64_t nr = last_logits_rows[which];
        if (nr * V > cap) { err = "output buffer too small"; return DFLASH_EINVAL; }
        dflash_status r = sync("debug_logits");
        if (r) return r;
        const float *src = which == 2 ? plogits : (which == 0 && c.sampling ? qlogits : logits);
        if (cudaMemcpy(out, src, sizeof(float) * nr * V, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("logits copy");
        if (rows) *rows = nr;
        return DFLASH_OK;
    }

    dflash_status seq_state(int seq, int32_t *len, int32_t *anchor, int32_t *n_out) override {
        if (seq < 0 || seq >= c.max_batch) { err = "bad slot"; return DFLASH_EINVAL; }
        dflash_status r = sync("seq_state");
        if (r) return r;
        SeqState hs;
        if (cudaMemcpy(&hs, st + seq, sizeof hs, cudaMemcpyDeviceToHost) != cudaSuccess) return fail_cuda("state copy");
        if (len) *len = hs.len;
        if (anchor) *anchor = hs.anchor;
        if (n_out) *n_out = hs.n_out;
        return DFLASH_OK;
    }

    dflash_status debug_kv(int which, int layer, int seq, int p0, int n, float *ko, float *vo) override {
        const dflash_model_cfg &m = which == 0 ? c.target : c.drafter;
        if (which < 0 || which > 1 || layer < 0 || layer >= m.n_layers || seq < 0 || seq >= c.max_batch || p0 < 0 ||
            n < 1 || p0 + n > c.max_len || !ko || !vo) {
            err = "bad debug_kv arguments";
            return DFLASH_EINVAL;
        }
        dflash_status r = sync("debug_kv");
        if (r) return r;
        const T *kc = (which == 0 ? tk : dk) + (size_t)layer * kv_layer_elems(m);
        const T *vc = (which == 0 ? tv : dv) + (size_t)layer * kv_layer_elems(m);
        const int hd = m.head_dim, nkv = m.n_kv_heads;
        std::vector<T> buf((size_t)n * hd), bl((size_t)n * hd);
        for (int pass = 0; pass < 2; ++pass) {
            const T *src = pass ? vc : kc;
            float *dst = pass ? vo : ko;
            for (int hh = 0; hh < nkv; ++hh) {
                const T *p = src + (((size_t)seq * nkv + hh) * c.max_len + p0) * hd;
                if (cudaMemcpy(buf.data(), p, sizeof(T) * n * hd, cudaMemcpyDeviceToHost) != cudaSuccess)
                    return fail_cuda("kv copy");
                if (lo_ && cudaMemcpy(bl.data(), p + lo_, sizeof(T) * n * hd, cudaMemcpyDeviceToHost) != cudaSuccess)
                    return fail_cuda("kv copy");
                for (int t = 0; t < n; ++t)
                    for (int e = 0; e < hd; ++e) {
                        const size_t i = (size_t)t * hd + e;
                        dst[(size_t)t * nkv * hd + hh * hd + e] = host_to_f(buf[i]) + (lo_ ? host_to_f(bl[i]) : 0.f);
                    }
            }
        }
        return DFLASH_OK;
    }

    static float host_to_f(float v) { return v; }
    static float host_to_f(bf16 v) {
        uint16_t b;
        memcpy(&b, &v, 2);
        uint32_t u = (uint32_t)b << 16;
        float f;
        memcpy(&f, &u, 4);
        return f;
    }

    dflash_status decode_iters(int n, int iters) override {
        if (n < 1 || n > c.max_batch || iters < 0) { err = "bad decode_iters arguments"; return DFLASH_EINVAL; }
        dflash_status r = refresh_lens();
        if (r) return r;
        for (int i = 0; i < n; ++i) {
            if (!h_prefilled[i]) { err = "slot not prefilled"; return DFLASH_ESTATE; }
            if ((int64_t)h_len[i] + (int64_t)(iters + 1) * c.block_size > c.max_len) {
                err = "decode_iters could exceed max_len";
                return DFLASH_ECAPACITY;
            }
        }
        std::vector<int32_t> iota(n);
        for (int i = 0; i < n; ++i) iota[i] = i;
        if ((r = set_active(iota.data(), n))) return r;
        OtherPass mark{last_pass};
        for (int it = 0; it < iters; ++it) {
            timed_pass(DFLASH_PROF_DRAFT_PASS, [&] { enqueue_draft(n, true); });
            timed_pass(DFLASH_PROF_VERIFY_PASS, [&] { enqueue_verify(n); });
        }
        last_draft.clear();
        lens_stale = true;
        return check("decode_iters launch");
    }

    dflash_status get_stats(dflash_stats *o) override {
        if (!o) { err = "null stats"; return DFLASH_EINVAL; }
        dflash_status r = sync("stats");
        if (r) return r;
        DevStats hs;
        if (cudaMemcpy(&hs, stats, sizeof hs, cudaMemcpyDeviceToHost) != cudaSuccess) return fail_cuda("stats copy");
        memset(o, 0, sizeof *o);
        o->iterations = (int64_t)hs.iterations;
        o->tokens = (int64_t)hs.tokens;
        for (int i = 0; i < DFLASH_MAX_BLOCK; ++i) o->accept_hist[i] = (int64_t)hs.hist[i];
        o->mean_tau = hs.iterations ? (double)hs.tokens / (double)hs.iterations : 0.0;
        o->kernel_launches = launch_count();
        return status_code(hs.status, err);
    }

    dflash_status reset_stats() override {
        if (cudaMemsetAsync(stats, 0, sizeof(DevStats), s) != cudaSuccess) return fail_cuda("stats reset");
        return DFLASH_OK;
    }

    dflash_status profile(int enable) override {
        dflash_status r = sync("profile");
        if (r) return r;
        if (enable < 0 || enable > 3) { err = "profile mode must be 0..3"; return DFLASH_EINVAL; }
        profiling = enable;
        if (profiling) {
            prof.clear();
            ev_used = 0;
        }
        return DFLASH_OK;
    }

    dflash_status profile_read(dflash_kernel_prof *o) override {
        if (!o) { err = "null profile output"; return DFLASH_EINVAL; }
        dflash_status r = sync("profile_read");
        if (r) return r;
        for (int k = 0; k < DFLASH_PROF_CLASSES; ++k) o[k] = dflash_kernel_prof{0, 0.0, 0.0};
        for (const ProfRec &p : prof) {
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) return fail_cuda("event time");
            for (int k : p.cls) {
                if (k < 0 || k >= DFLASH_PROF_CLASSES) continue;
                o[k].launches += 1;
                o[k].ms += ms;
                o[k].bytes += p.bytes;
            }
        }
        return DFLASH_OK;
    }

    // LM-head argmax of the rows of the last pass, with the per-tile partials
    // and the output ids in caller-free static scratch (see dflash.h).
    dflash_status head_argmax_noalloc(int which, int32_t *host_out, int32_t *rows_out, void *scratch) override {
        if (!std::is_same<T, bf16>::value) { err = "dflash_head_argmax_noalloc needs a bf16 context"; return DFLASH_EUNSUPPORTED; }
        if (which < 0 || which > 2 || !host_out || !rows_out) { err = "bad dflash_head_argmax_noalloc arguments"; return DFLASH_EINVAL; }
        const int V = c.target.vocab, H = c.target.hidden, B = c.block_size;
        if (last_pass != which) {
            err = "the last pass on this context is not of the requested kind (call right after that pass)";
            return DFLASH_ESTATE;
        }
        if (sampling_on() || (which == 0 && draft_mode == DFLASH_DRAFT_SCRIPT)) {
            err = "dflash_head_argmax_noalloc returns greedy argmaxes: not with sampling or script drafts";
            return DFLASH_ESTATE;
        }
        const int rows = last_logits_rows[which];
        const int n_tiles = (V + 127) / 128;
        if (rows < 1) { err = "no pass of that kind has run on this context"; return DFLASH_ESTATE; }
        if (rows > kNoallocRows || n_tiles > kNoallocTiles) {
            err = "dflash_head_argmax_noalloc: more than 64 rows or a vocabulary above 262144";
            return DFLASH_ECAPACITY;
        }
        float2 *part = reinterpret_cast<float2 *>(scratch);
        int *idx = reinterpret_cast<int *>(reinterpret_cast<char *>(scratch) + kNoallocPartBytes);
        Epi<T> e;
        e.kind = EPI_LOGITS;
        e.Y = nullptr;
        e.ldy = V;
        float2 *saved_part = tc.lm_part;
        const int saved_keep = tc.keep_logits;
        tc.lm_part = part;
        tc.keep_logits = 0;
        int ctas = 0;
        if (which < 2 && fold_used[which]) {
            // folded passes feed the head bf16(x * g_final) and scale each row by its RMSNorm factor
            const float eps = (float)(which == 0 ? c.drafter.rms_eps : c.target.rms_eps);
            ctas = gemm_launch(xg_t, H, rows, lm_head, V, H, epi_norm_in(e, eps, H), nullptr, 0, nullptr,
                               scales_of(lm_head));
        } else {
            ctas = gemm_launch(xn, H, rows, lm_head, V, H, e, nullptr, 0, nullptr, scales_of(lm_head));
        }
        tc.lm_part = saved_part;
        tc.keep_logits = saved_keep;
        if (ctas < 1) {  // every partial the argmax reads must come from this call
            err = "dflash_head_argmax_noalloc: LM-head projection not launched: " + tc.err;
            return DFLASH_ECUDA;
        }
        const int mode = which == 0 ? 1 : 0;
        launch_lm_argmax(part, n_tiles, rows, mode, B, idx, nullptr, s);
        const int n_out = which == 0 ? (rows / B) * (B - 1) : rows;
        dflash_status r = sync("head_argmax_noalloc");
        if (r) return r;
        if (n_out > 0 && cudaMemcpy(host_out, idx, sizeof(int32_t) * n_out, cudaMemcpyDeviceToHost) != cudaSuccess)
            return fail_cuda("head_argmax_noalloc copy");
        *rows_out = n_out;
        return DFLASH_OK;
    }

    dflash_status set_script(int seq, const int32_t *sc, int n) override {
        if (seq < 0 || seq >= c.max_batch || !sc || n < 1 || n > c.max_len) { err = "bad script arguments"; return DFLASH_EINVAL; }
        for (int i = 0; i < n; ++i)
            if (sc[i] < 0 || sc[i] >= c.target.vocab) { err = "script id out of vocab"; return DFLASH_EINVAL; }
        if (cudaMemcpyAsync(script + (size_t)seq * c.max_len, sc, sizeof(int32_t) * n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return fail_cuda("script copy");
        return sync("script");
    }
};

}  // namespace dfl

using namespace dfl;

// ------------------------------------------------------------------------
// C ABI
// ------------------------------------------------------------------------

// Every call runs with the context's device current (restored on return), so
// one host thread can drive contexts on several devices.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
        else prev = -1;
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

extern "C" {

dflash_status dflash_workspace_size(const dflash_config *cfg, size_t *wb, size_t *sb) {
    if (!cfg || !wb || !sb) return DFLASH_EINVAL;
    std::string why;
    if (!check_config(*cfg, why)) return DFLASH_EINVAL;
    Layout L = make_layout(*cfg);
    *wb = L.weight_bytes;
    *sb = L.state_bytes;
    return DFLASH_OK;
}

dflash_status dflash_create(const dflash_config *cfg, void *warena, size_t wbytes, void *sarena, size_t sbytes,
                            void *stream, dflash_ctx **out) {
    if (!cfg || !out) return DFLASH_EINVAL;
    *out = nullptr;
    std::string why;
    if (!check_config(*cfg, why)) return DFLASH_EINVAL;
    dflash_ctx *ctx = new dflash_ctx();
    ctx->cfg = *cfg;
    ctx->lay = make_layout(*cfg);
    if (!warena || !sarena || wbytes < ctx->lay.weight_bytes || sbytes < ctx->lay.state_bytes ||
        ((uintptr_t)warena & 255) || ((uintptr_t)sarena & 255)) {
        delete ctx;
        return DFLASH_EINVAL;
    }
    for (size_t i = 0; i < ctx->lay.slots.size(); ++i) ctx->by_name[ctx->lay.slots[i].name] = (int)i;
    if (cudaGetDevice(&ctx->device) != cudaSuccess) {
        delete ctx;
        return DFLASH_ECUDA;
    }
    cudaStream_t s = (cudaStream_t)stream;
    if (cfg->dtype != DFLASH_FP32)
        ctx->eng.reset(new Engine<bf16>(*cfg, ctx->lay, (char *)warena, (char *)sarena, s));
    else
        ctx->eng.reset(new Engine<float>(*cfg, ctx->lay, (char *)warena, (char *)sarena, s));
    dflash_status r;
    if (cfg->dtype != DFLASH_FP32) r = static_cast<Engine<bf16> *>(ctx->eng.get())->init(ctx->by_name);
    else r = static_cast<Engine<float> *>(ctx->eng.get())->init(ctx->by_name);
    if (r != DFLASH_OK) {
        fprintf(stderr, "dflash_create: %s\n", ctx->eng->err.c_str());
        delete ctx;
        return r;
    }
    *out = ctx;
    return DFLASH_OK;
}

void dflash_destroy(dflash_ctx *ctx) {
    if (!ctx) return;
    DeviceGuard g(ctx->device);
    delete ctx;
}

const char *dflash_last_error(const dflash_ctx *ctx) {
    if (!ctx) return "null context";
    return ctx->err.c_str();
}

int32_t dflash_weight_count(const dflash_ctx *ctx) { return ctx ? (int32_t)ctx->lay.slots.size() : 0; }

dflash_status dflash_weight_info(const dflash_ctx *ctx, int32_t i, const char **name, size_t *offset, size_t *numel,
                                 int32_t *dtype, int32_t *ndim, int64_t *shape) {
    if (!ctx || i < 0 || i >= (int32_t)ctx->lay.slots.size()) return DFLASH_EINVAL;
    const WeightSlot &w = ctx->lay.slots[i];
    if (name) *name = w.name.c_str();
    if (offset) *offset = w.offset;
    if (numel) *numel = w.numel;
    if (dtype) *dtype = w.dtype;
    if (ndim) *ndim = w.ndim;
    if (shape) for (int k = 0; k < 3; ++k) shape[k] = w.shape[k];
    return DFLASH_OK;
}

dflash_status dflash_weight_slot(const dflash_ctx *ctx, const char *name, size_t *offset, size_t *numel,
                                 int32_t *dtype) {
    if (!ctx || !name) return DFLASH_EINVAL;
    auto it = ctx->by_name.find(name);
    if (it == ctx->by_name.end()) return DFLASH_EINVAL;
    const WeightSlot &w = ctx->lay.slots[it->second];
    if (offset) *offset = w.offset;
    if (numel) *numel = w.numel;
    if (dtype) *dtype = w.dtype;
    return DFLASH_OK;
}

#define DFL_CALL(ctx, expr)                                                   \
    do {                                                                      \
        if (!(ctx)) return DFLASH_EINVAL;                                     \
        if ((ctx)->broken) { (ctx)->err = "context unusable after a CUDA error"; return DFLASH_ECUDA; } \
        DeviceGuard _dg((ctx)->device);                                       \
        if (!_dg.ok) { (ctx)->err = "cannot make the context's device current"; return DFLASH_ECUDA; } \
        dflash_status _r = (expr);                                            \
        (ctx)->err = _r ? (ctx)->eng->err : std::string();                    \
        if (_r == DFLASH_ECUDA) (ctx)->broken = true;                         \
        return _r;                                                            \
    } while (0)

dflash_status dflash_prefill(dflash_ctx *ctx, int32_t seq, const int32_t *prompt, int32_t n, int32_t *first) {
    DFL_CALL(ctx, ctx->eng->prefill(seq, prompt, n, INT_MAX, first));
}

dflash_status dflash_draft_block(dflash_ctx *ctx, const int32_t *seqs, int32_t n, int32_t *drafts) {
    DFL_CALL(ctx, ctx->eng->draft(seqs, n, drafts, drafts != nullptr));
}

dflash_status dflash_verify_commit(dflash_ctx *ctx, const int32_t *seqs, int32_t n, const int32_t *drafts,
                                   int32_t *accept, int32_t *committed, int32_t *new_len) {
    DFL_CALL(ctx, ctx->eng->verify(seqs, n, drafts, accept, committed, new_len));
}

dflash_status dflash_generate(dflash_ctx *ctx, const int32_t *const *prompts, const int32_t *lens, int32_t n,
                              int32_t max_new, int32_t *out, dflash_stats *stats) {
    if (!out) return DFLASH_EINVAL;
    DFL_CALL(ctx, ctx->eng->generate(prompts, lens, n, max_new, out, stats));
}

dflash_status dflash_generate_ar(dflash_ctx *ctx, const int32_t *const *prompts, const int32_t *lens, int32_t n,
                                 int32_t max_new, int32_t *out, double *ms) {
    if (!out) return DFLASH_EINVAL;
    DFL_CALL(ctx, ctx->eng->generate_ar(prompts, lens, n, max_new, out, ms));
}

dflash_status dflash_decode_iters(dflash_ctx *ctx, int32_t n, int32_t iters) {
    DFL_CALL(ctx, ctx->eng->decode_iters(n, iters));
}

dflash_status dflash_get_stats(dflash_ctx *ctx, dflash_stats *out) { DFL_CALL(ctx, ctx->eng->get_stats(out)); }

dflash_status dflash_reset_stats(dflash_ctx *ctx) { DFL_CALL(ctx, ctx->eng->reset_stats()); }

dflash_status dflash_profile(dflash_ctx *ctx, int32_t enable) { DFL_CALL(ctx, ctx->eng->profile(enable)); }

dflash_status dflash_profile_read(dflash_ctx *ctx, dflash_kernel_prof *out) {
    DFL_CALL(ctx, ctx->eng->profile_read(out));
}

dflash_status dflash_head_argmax_noalloc(dflash_ctx *ctx, int32_t which, int32_t *host_out, int32_t *rows_out) {
    if (!ctx) return DFLASH_EINVAL;
    if (ctx->broken) {
        ctx->err = "context unusable after a CUDA error";
        return DFLASH_ECUDA;
    }
    std::string e;
    void *scratch = noalloc_scratch_ptr(ctx->device, e);
    if (!scratch) {
        ctx->err = e;
        return DFLASH_ECUDA;
    }
    DFL_CALL(ctx, ctx->eng->head_argmax_noalloc(which, host_out, rows_out, scratch));
}

dflash_status dflash_set_draft_mode(dflash_ctx *ctx, int32_t mode, int32_t tau) {
    if (!ctx) return DFLASH_EINVAL;
    if ((mode != DFLASH_DRAFT_MODEL && mode != DFLASH_DRAFT_SCRIPT) || tau < 1 || tau > ctx->cfg.block_size)
        return DFLASH_EINVAL;
    if (mode == DFLASH_DRAFT_SCRIPT && ctx->eng->temperature > 0.f) {
        ctx->err = "script drafts are for greedy decoding (temperature is above 0)";
        return DFLASH_ESTATE;
    }
    ctx->eng->draft_mode = mode;
    ctx->eng->tau = tau;
    return DFLASH_OK;
}

dflash_status dflash_set_sampling(dflash_ctx *ctx, double temperature, uint64_t seed) {
    if (!ctx) return DFLASH_EINVAL;
    if (!(temperature >= 0.0) || temperature > 1e30) {
        ctx->err = "temperature must be a finite number >= 0";
        return DFLASH_EINVAL;
    }
    if (temperature > 0.0 && !ctx->cfg.sampling) {
        ctx->err = "context created without sampling";
        return DFLASH_ESTATE;
    }
    if (temperature > 0.0 && ctx->eng->draft_mode == DFLASH_DRAFT_SCRIPT) {
        ctx->err = "script drafts are for greedy decoding";
        return DFLASH_ESTATE;
    }
    ctx->eng->temperature = (float)temperature;
    ctx->eng->seed = seed;
    ctx->eng->sampling_changed();
    ctx->err.clear();
    return DFLASH_OK;
}

dflash_status dflash_set_script(dflash_ctx *ctx, int32_t seq, const int32_t *script, int32_t n) {
    DFL_CALL(ctx, ctx->eng->set_script(seq, script, n));
}

dflash_status dflash_debug_logits(dflash_ctx *ctx, int32_t which, float *out, int64_t cap, int64_t *rows) {
    DFL_CALL(ctx, ctx->eng->debug_logits(which, out, cap, rows));
}

dflash_status dflash_seq_state(dflash_ctx *ctx, int32_t seq, int32_t *len, int32_t *anchor, int32_t *n_out) {
    DFL_CALL(ctx, ctx->eng->seq_state(seq, len, anchor, n_out));
}

dflash_status dflash_debug_kv(dflash_ctx *ctx, int32_t which, int32_t layer, int32_t seq, int32_t p0, int32_t n,
                              float *k, float *v) {
    DFL_CALL(ctx, ctx->eng->debug_kv(which, layer, seq, p0, n, k, v));
}

}  // extern "C"
