// engine.h -- internal structures of a dflash context.
#pragma once

#include <memory>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/dflash.h"
#include "kernels.h"

namespace dfl {

constexpr int kMaxDevices = 64;

struct WeightSlot {
    std::string name;
    size_t offset = 0, numel = 0;
    int dtype = 0;  // DFLASH_FP32 / DFLASH_BF16 / DFLASH_FP8 / DFLASH_FP4 / DFLASH_UE8M0
    int ndim = 0;
    int64_t shape[3] = {0, 0, 0};
};

// Scales of a quantised projection matrix (from row blk_row0 on): FP8 / FP4 row
// scales; FP4 block exponents [K/128][blk_rows][4] of the whole matrix
struct WScales {
    const float *row = nullptr;
    const uint8_t *blk = nullptr;
    int blk_rows = 0, blk_row0 = 0;
};

struct LayerW {
    const float *attn_norm = nullptr, *ffn_norm = nullptr;
    const float *q_norm = nullptr, *k_norm = nullptr;  // QK-norm gains (fidelity toggle)
    const void *wqkv = nullptr, *wo = nullptr, *w_gate_up = nullptr, *w_down = nullptr;
    const void *w_router = nullptr, *we_gate_up = nullptr, *we_down = nullptr;
};

// Byte layout of the two arenas, computed identically by workspace_size and create.
struct Layout {
    std::vector<WeightSlot> slots;
    size_t weight_bytes = 0;
    // state arena offsets
    size_t x, xn, dq_in, Y, q, ao, h, taps_dec, taps_gather, taps_pre, cbuf, logits, plogits;
    size_t qlogits, lse_p, lse_q, samp_part, tok_p, resid;  // temperature sampling (config.sampling)
    size_t g, drafts, accept, committed, new_len, st, active, meta, ctx_meta, ctx_meta_pre;
    size_t rope_t, rope_d, tk, tv, dk, dv, script, out_tok, tokens, stats, first_tok;
    size_t moe_sel, moe_wt, moe_part, moe_off = 0, moe_list = 0, moe_xg = 0, lm_part, att_o, att_ml, att_sem;
    size_t att_parts = 0;
    size_t xg_t, xg2, ssq, dep_v, dep_d;
    size_t mx_codes = 0, mx_words = 0;  // FP8: MX planes of a projection's activation rows
    int mx_mpad = 0, mx_kpad = 0;
    size_t act_lo = 0;  // two-plane activations: low plane offset in elements (0: one plane)
    int ssq_ld = 0, n_ops_v = 0, n_ops_d = 0;
    size_t gemm_ws, gemm_sem;
    size_t state_bytes = 0;
    // dims
    int R_dec = 0, C = 0, R_max = 0, Y_cols = 0, ws_floats = 0, n_sem = 0;
};

struct Status {
    dflash_status code;
    std::string msg;
};

class EngineBase {
  public:
    virtual ~EngineBase() {}
    virtual dflash_status prefill(int seq, const int32_t *prompt, int n, int max_new, int32_t *first) = 0;
    virtual dflash_status draft(const int32_t *seqs, int n, int32_t *drafts, bool sync) = 0;
    virtual dflash_status verify(const int32_t *seqs, int n, const int32_t *drafts, int32_t *accept,
                                 int32_t *committed, int32_t *new_len) = 0;
    virtual dflash_status generate(const int32_t *const *prompts, const int32_t *lens, int n, int max_new,
                                   int32_t *out, dflash_stats *stats) = 0;
    virtual dflash_status generate_ar(const int32_t *const *prompts, const int32_t *lens, int n,
                                      int max_new, int32_t *out, double *ms) = 0;
    virtual dflash_status debug_logits(int which, float *out, int64_t cap, int64_t *rows) = 0;
    virtual dflash_status seq_state(int seq, int32_t *len, int32_t *anchor, int32_t *n_out) = 0;
    virtual dflash_status debug_kv(int which, int layer, int seq, int p0, int n, float *k, float *v) = 0;
    virtual dflash_status set_script(int seq, const int32_t *script, int n) = 0;
    virtual dflash_status decode_iters(int n, int iters) = 0;
    virtual dflash_status get_stats(dflash_stats *out) = 0;
    virtual dflash_status reset_stats() = 0;
    virtual dflash_status profile(int enable) = 0;
    virtual dflash_status profile_read(dflash_kernel_prof *out) = 0;
    virtual dflash_status head_argmax_noalloc(int which, int32_t *host_out, int32_t *rows_out, void *scratch) = 0;
    virtual void sampling_changed() {}
    std::string err;
    int draft_mode = DFLASH_DRAFT_MODEL, tau = 1;
    float temperature = 0.f;  // > 0: temperature sampling (config.sampling), else greedy
    uint64_t seed = 0;
};

}  // namespace dfl

struct dflash_ctx {
    dflash_config cfg;
    dfl::Layout lay;
    std::unordered_map<std::string, int> by_name;
    std::unique_ptr<dfl::EngineBase> eng;
    std::string err;
    bool broken = false;
    int device = 0;  // CUDA device the context was created on
};
