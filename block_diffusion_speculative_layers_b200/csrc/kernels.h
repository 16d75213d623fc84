// kernels.h -- host launchers of the DFlash kernels (internal interface).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "philox.cuh"

namespace dfl {

// Host-side count of kernels launched by this library (all contexts).
void note_launch();
long long launch_count();

// Tap destinations of one target layer: the residual after the layer is
// copied (rounded to T) to columns col[i] .. col[i]+H of row meta[r].aux of
// `base` (leading dimension ld), for i < n.
template <typename T>
struct TapDst {
    T *base;
    int ld;
    int n;
    int col[8];
};

// ---- rows: embedding + metadata ----
template <typename T>
void launch_embed_block(const T *emb, int H, SeqState *st, const int *active, int nseq, int B,
                        int is_draft, const int *drafts, int mask_id, float *x, RowMeta *meta,
                        RowMeta *ctx_meta, cudaStream_t s);
template <typename T>
void launch_embed_norm(const T *emb, int H, SeqState *st, const int *active, int nseq, int B, int is_draft,
                       const int *drafts, int mask_id, float *x, RowMeta *meta, RowMeta *ctx_meta, const float *g, T *xg,
                       int xg_ld, size_t lo, float *ssq, int ssq_ld, cudaStream_t s);
template <typename T>
void launch_embed_tokens(const T *emb, int H, const int *tokens, int R, int seq, int pos0,
                         float *x, RowMeta *meta, cudaStream_t s);
void launch_ctx_meta_prefill(RowMeta *meta, int R, int seq, int pos0, cudaStream_t s);

// ---- normalisation / elementwise ----
// `lo` (elements) is the offset of the low plane of two-plane bf16 activations
// (see st_act in common.cuh); 0 for single-plane outputs.
template <typename TO>
void launch_rmsnorm(const float *x, int ldx, const float *g, int H, float eps, TO *out, int ldo, size_t lo,
                    int R, cudaStream_t s);
template <typename T>
void launch_residual(float *x, const float *Y, int ldy, int H, int R, const TapDst<T> &taps, size_t lo,
                     const RowMeta *meta, cudaStream_t s);
template <typename T>
void launch_swiglu(const float *Y, int ldy, int F, int R, T *h, int ldh, size_t lo, cudaStream_t s);
template <typename T>
void launch_qkv_epilogue(const float *Y, int ldy, int col0, int R_blk, int R_tot,
                         const RowMeta *meta, const RowMeta *ctx_meta, int nq, int nkv, int hd,
                         const float2 *rope, T *q_out, T *kc, T *vc, int max_len, size_t lo, const float *qn_g,
                         const float *kn_g, float qk_eps, cudaStream_t s);

// ---- GEMM (CUDA-core, fp32 accumulate): Y[M][N] = X[M][K] . W[N][K]^T ----
template <typename T>
void launch_gemm_simt(const T *X, int ldx, int M, const T *W, int ldw, int N, int K, float *Y,
                      int ldy, size_t lo, cudaStream_t s);

// ---- attention (CUDA-core reference path, used for fp32 models) ----
template <typename T>
void launch_attention_simt(const T *q, int ldq, const T *kc, const T *vc, const RowMeta *meta,
                           int R, int nq, int nkv, int hd, int max_len, T *out, int ldo,
                           cudaStream_t s);

// ---- heads, acceptance, scripts ----
// mode 0: idx[r] = argmax of row r.  mode 1 (drafter): rows r = i*B + j with
// j >= 1 go to idx[i*(B-1) + j-1]; rows with j == 0 are skipped.
void launch_argmax_rows(const float *logits, int64_t ldl, int V, int R, int mode, int B, int *idx,
                        DevStats *stats, cudaStream_t s);
void launch_accept(SeqState *st, const int *active, int nseq, int B, const int *drafts,
                   const int *g, int *accept, int *committed, int *new_len, int *out_tok,
                   int out_ld, DevStats *stats, cudaStream_t s);
void launch_script_drafts(const SeqState *st, const int *active, int nseq, int B, int tau, int V,
                          const int *script, int script_ld, int *drafts, cudaStream_t s);
void launch_prefill_finish(SeqState *st, int seq, int n, const int *first_tok, int *out_tok,
                           int out_ld, int max_new, cudaStream_t s);
void launch_ar_step(SeqState *st, const int *active, int nseq, const int *g, int *out_tok,
                    int out_ld, DevStats *stats, cudaStream_t s);

// ---- MoE (routing + CUDA-core expert FFN reference path) ----
void launch_moe_topk(const float *router_logits, int E, int R, int k, int *sel, float *wt,
                     cudaStream_t s);
template <typename T>
void launch_moe_experts_simt(const T *m, int ldm, size_t lo, int R, int k, const int *sel, const T *w_gate_up,
                             const T *w_down, int H, int Fe, float *part, cudaStream_t s);
// Bucketed experts (bf16, moe_experts.cu): pairs grouped by expert (off[2E+2]:
// pair ranges then the touched-expert list; list[R*k] scratch), then gate/up ->
// h[pair][Fe] (two planes when hlo != 0) and down -> part[pair][H], each a
// persistent weight-streaming kernel of num_sms CTAs; timed-out waits set bit 4 of *err.
bool moe_bucketed_supported(int H, int Fe, int E);
// Rows of the pairs in expert-grouped order: xg[pos] = m[list[pos] / k] (both
// planes), for the grouped tensor-core expert projections.
void launch_moe_gather(const bf16 *m, int ldm, size_t lo, const int *list, int k, int n_pairs, int H, bf16 *xg,
                       cudaStream_t s);
// Bucketing alone: off[E+1] pair ranges, list[n_pairs] pairs by expert, off[E+1 ..
// 2E+1] touched experts (ascending, -1 after them), off[2E+1] their count.
void launch_moe_bucket(const int *sel, int n_pairs, int E, int *off, int *list, cudaStream_t s);
void launch_moe_experts_bucketed(const bf16 *m, int ldm, size_t lo, int R, int k, const int *sel, int E,
                                 const bf16 *w_gate_up, const bf16 *w_down, int H, int Fe, int *off, int *list,
                                 bf16 *h, size_t hlo, float *part, int num_sms, int *err, cudaStream_t s);
template <typename T>
void launch_moe_combine(float *x, const float *part, const float *wt, int H, int R, int k,
                        const TapDst<T> &taps, size_t lo, const RowMeta *meta, cudaStream_t s);

// ---- temperature sampling (sampling.cu) ----
// Rows of fp32 logits -> per-row log-sum-exp of z/T and a Gumbel-max draw from
// softmax(z/T); draw positions: fixed_pos (one row, slot fixed_slot, prefill)
// or st[active[i]].len + k + pos_off for row k of sequence i.
struct SampleRows {
    const float *logits = nullptr;
    int ldl = 0, V = 0, R = 0, B = 1;
    int mode = 0;  // 0: every row -> tok[r]; 1: block rows k >= 1 -> tok[i*(B-1)+k-1] (drafts)
    float inv_T = 1.f;
    SampleKey key{0, 0};
    uint32_t purpose = SP_TARGET;
    int pos_off = 0, fixed_pos = -1, fixed_slot = -1;
    const SeqState *st = nullptr;
    const int *active = nullptr;
    float4 *part = nullptr;  // [sample_chunks(V)][R] scratch
    float *lse = nullptr;    // [R] or null
    int *tok = nullptr;
    DevStats *stats = nullptr;
};
// Residual draws from max(0, P_{k-1} - Q_k) for block positions k = 1..B-1 of
// every sequence: plog/qlog rows i*B+k-1 / i*B+k, resid[i*(B-1)+k-1] (-1: none).
struct ResidualRows {
    const float *plog = nullptr, *qlog = nullptr;
    int ldl = 0, V = 0, B = 1, rows = 0;
    float inv_T = 1.f;
    SampleKey key{0, 0};
    const float *lse_p = nullptr, *lse_q = nullptr;
    const SeqState *st = nullptr;
    const int *active = nullptr;
    float2 *part = nullptr;  // [sample_chunks(V)][rows] scratch
    int *resid = nullptr;
};
// The speculative-sampling acceptance + commit, one thread per sequence.
struct AcceptSample {
    SeqState *st = nullptr;
    const int *active = nullptr;
    int nseq = 0, B = 1;
    const int *drafts = nullptr;
    const float *plog = nullptr, *qlog = nullptr;
    int ldl = 0;
    const float *lse_p = nullptr, *lse_q = nullptr;
    float inv_T = 1.f;
    SampleKey key{0, 0};
    const int *resid = nullptr, *tok_p = nullptr;  // residual draws; target draws (row B-1: the bonus)
    int *accept = nullptr, *committed = nullptr, *new_len = nullptr, *out_tok = nullptr;
    int out_ld = 0;
    DevStats *stats = nullptr;
};
int sample_chunks(int V);
void launch_sample_rows(const SampleRows &a, cudaStream_t s);
void launch_residual_rows(const ResidualRows &a, cudaStream_t s);
void launch_accept_sample(const AcceptSample &a, cudaStream_t s);

// ---- tables ----
// (cos, sin) of position x frequency for every position and RoPE pair, in fp64;
// factor > 1: the frequencies rescaled in the Llama 3.1 form (low / high
// frequency factors, original maximum position).
void launch_rope_table(float2 *tab, int max_len, int hd, double theta, double factor, double low, double high,
                       double orig, cudaStream_t s);

}  // namespace dfl

namespace dfl {

// Epilogue of a projection Y[M][N] = X[M][K] . W[N][K]^T.
enum EpiKind { EPI_STORE = 0, EPI_QKV = 1, EPI_RESID = 2, EPI_SWIGLU = 3, EPI_LOGITS = 4, EPI_NORMOUT = 5 };

template <typename T>
struct Epi {
    EpiKind kind = EPI_STORE;
    // EPI_STORE / EPI_LOGITS: fp32 output Y[M][ldy]
    float *Y = nullptr;
    int ldy = 0;
    // EPI_STORE: output row of activation row m is row_map[m] (nullptr: m)
    const int *row_map = nullptr;
    // EPI_QKV: columns are rows col0.. of [Wq; Wk; Wv]; rows < R_blk are block rows
    // (q, k, v at meta.pos), rows >= R_blk context rows (k, v at ctx_meta.pos if aux)
    int col0 = 0, R_blk = 0;
    const RowMeta *meta = nullptr, *ctx_meta = nullptr;
    int nq = 0, nkv = 0, hd = 0, max_len = 0;
    const float2 *rope = nullptr;
    T *q_out = nullptr, *kc = nullptr, *vc = nullptr;
    // QK-norm (qn_g != nullptr): q and k heads RMS-normalised over hd with these
    // gains and qk_eps before RoPE
    const float *qn_g = nullptr, *kn_g = nullptr;
    float qk_eps = 0.f;
    // EPI_RESID: x[M][N] += Y, then tap copies of the new x
    float *x = nullptr;
    TapDst<T> taps{};
    // EPI_SWIGLU: N = 2F, columns [gate; up]; h[M][F] = SiLU(gate) * up
    T *h = nullptr;
    int F = 0;
    // RMSNorm folded into the projection.  Consumer side (QKV, SwiGLU, logits,
    // store): the input rows are bf16(x * g) and the result of row m is scaled
    // by 1/sqrt(sum_t rs_ssq[t*rs_ld + m] * rs_inv_n + rs_eps).
    const float *rs_ssq = nullptr;
    int rs_tiles = 0, rs_ld = 0;
    float rs_inv_n = 0.f, rs_eps = 0.f;
    // Producer side (EPI_RESID after the add, EPI_NORMOUT on the raw result y):
    // xg[m][n] = bf16(y[m][n] * g_next[n]) and ssq_out[tile*ssq_ld + m] =
    // sum of y^2 over the tile's 128 columns (for the next projection's norm).
    T *xg = nullptr;
    int xg_ld = 0;
    const float *g_next = nullptr;
    float *ssq_out = nullptr;
    int ssq_ld = 0;
    // two-plane bf16 activations: offset (elements) of the low plane of the
    // input X and of every T output above (q_out, kc, vc, taps, h, xg); 0 = one plane
    size_t lo = 0;
};

void launch_gather_rows(const void *src, void *dst, size_t row_bytes, const int *active, int nseq, int B,
                        cudaStream_t s);

}  // namespace dfl
