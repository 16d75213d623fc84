// kernels_rows.cu -- row bookkeeping, normalisation, elementwise epilogues,
// greedy heads and the accept/commit step of the DFlash decode iteration.
//
// Method passages (DFlash pages, by title and section):
//  * "DFlash: Decodificação Especulativa com Blocos em Paralelo ..." (iaemfoco),
//    "O que o DFlash faz de diferente": the drafter fills a whole block in one
//    pass; the target verifies the block in parallel.  Block rows are
//    [anchor, mask x (B-1)] for the drafter and [anchor, d_1..d_{B-1}] for
//    the target.
//  * same page, "Decodificação especulativa tradicional": accepted tokens are
//    kept and the output equals target-only decoding -> greedy acceptance of
//    the longest prefix with d_i == g_{i-1}, plus the target's bonus token.
//  * "Nova técnica faz modelo Qwen rodar ..." (forbuilders), "Como funciona a
//    decodificação especulativa": only the wrong entries are discarded -> the
//    KV cache is rolled back by length only.
#include <math.h>

#include <atomic>

#include "kernels.h"
#include "launch.h"

namespace dfl {

static std::atomic<long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
long long launch_count() { return g_launches.load(std::memory_order_relaxed); }

// ------------------------------------------------------------------------
// embeddings + row metadata
// ------------------------------------------------------------------------

// x[0..H) = float(e[0..H)) with 16-byte loads, all issued before any store
// (H a multiple of 64, rows 16-byte aligned).
template <typename T>
__device__ __forceinline__ void copy_embedding_row(const T *__restrict__ e, float *__restrict__ xr, int H) {
    constexpr int EPC = 16 / (int)sizeof(T);
    constexpr int NV = 4;
    const uint4 *e4 = reinterpret_cast<const uint4 *>(e);
    const int nch = H / EPC;
    for (int base = 0; base < nch; base += NV * blockDim.x) {
        uint4 raw[NV];
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int ch = base + threadIdx.x + u * blockDim.x;
            raw[u] = ch < nch ? e4[ch] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int ch = base + threadIdx.x + u * blockDim.x;
            if (ch >= nch) continue;
            const T *vals = reinterpret_cast<const T *>(&raw[u]);
#pragma unroll
            for (int k = 0; k < EPC; ++k) xr[ch * EPC + k] = to_f(vals[k]);
        }
    }
}

template <typename T>
__global__ void embed_block_kernel(const T *__restrict__ emb, int H, SeqState *st,
                                   const int *__restrict__ active, int B, int is_draft,
                                   const int *__restrict__ drafts, int mask_id, float *__restrict__ x,
                                   RowMeta *meta, RowMeta *ctx_meta) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int i = r / B, j = r % B;
    const int s = active[i];
    const SeqState S = st[s];
    const int p = S.len;
    int tok;
    if (j == 0) tok = S.anchor;
    else tok = is_draft ? mask_id : drafts[i * (B - 1) + (j - 1)];
    copy_embedding_row(emb + (size_t)tok * H, x + (size_t)r * H, H);
    if (threadIdx.x == 0) {
        RowMeta m;
        m.seq = s;
        m.pos = p + j;
        m.nk = is_draft ? p + B : p + j + 1;
        m.aux = s * B + j;  // pending tap row of the slot
        meta[r] = m;
        if (is_draft && ctx_meta) {
            RowMeta c;
            c.seq = s;
            c.pos = S.pend_pos0 + j;
            c.nk = 0;
            c.aux = (j < S.pend_n) ? 1 : 0;
            ctx_meta[r] = c;
        }
    }
}

template <typename T>
void launch_embed_block(const T *emb, int H, SeqState *st, const int *active, int nseq, int B,
                        int is_draft, const int *drafts, int mask_id, float *x, RowMeta *meta,
                        RowMeta *ctx_meta, cudaStream_t s) {
    launch_k(embed_block_kernel<T>, dim3(nseq * B), dim3(256), 0, s, 1, emb, H, st, active, B, is_draft, drafts, mask_id,
                                                   x, meta, ctx_meta);
}

// Block rows as embed_block_kernel, plus the folded RMSNorm inputs of the first
// projection: xg = x * g (two planes when lo != 0) and per-128-column-tile sums
// of squares.  Each thread loads its 16-byte chunks of the embedding row
// before using any of them, so a row costs one memory latency, not one per column.
template <typename T>
__global__ void embed_norm_kernel(const T *__restrict__ emb, int H, SeqState *st, const int *__restrict__ active, int B,
                                  int is_draft, const int *__restrict__ drafts, int mask_id, float *__restrict__ x,
                                  RowMeta *meta, RowMeta *ctx_meta, const float *__restrict__ g, T *__restrict__ xg,
                                  int xg_ld, size_t lo, float *__restrict__ ssq, int ssq_ld) {
    pdl_trigger();
    pdl_wait();
    constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    constexpr int CPT = 128 / EPC;            // chunks per 128-column tile (divides 32)
    constexpr int NV = 4;                     // chunks in flight per thread
    const int r = blockIdx.x;
    const int i = r / B, j = r % B;
    const int s = active[i];
    const SeqState S = st[s];
    const int p = S.len;
    const int tok = j == 0 ? S.anchor : (is_draft ? mask_id : drafts[i * (B - 1) + (j - 1)]);
    const uint4 *e4 = reinterpret_cast<const uint4 *>(emb + (size_t)tok * H);
    const int nch = H / EPC;
    for (int base = 0; base < nch; base += NV * blockDim.x) {
        uint4 raw[NV];
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int ch = base + threadIdx.x + u * blockDim.x;
            raw[u] = ch < nch ? e4[ch] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int ch = base + threadIdx.x + u * blockDim.x;
            const T *vals = reinterpret_cast<const T *>(&raw[u]);
            float sq = 0.f;
            if (ch < nch) {
#pragma unroll
                for (int k = 0; k < EPC; ++k) {
                    const int col = ch * EPC + k;
                    const float v = to_f(vals[k]);
                    x[(size_t)r * H + col] = v;
                    st_act(xg, (size_t)r * xg_ld + col, lo, v * g[col]);
                    sq += v * v;
                }
            }
#pragma unroll
            for (int o = CPT / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (ch < nch && (threadIdx.x % CPT) == 0) ssq[(size_t)(ch / CPT) * ssq_ld + r] = sq;
        }
    }
    if (threadIdx.x == 0) {
        RowMeta m;
        m.seq = s;
        m.pos = p + j;
        m.nk = is_draft ? p + B : p + j + 1;
        m.aux = s * B + j;
        meta[r] = m;
        if (is_draft && ctx_meta) {
            RowMeta c;
            c.seq = s;
            c.pos = S.pend_pos0 + j;
            c.nk = 0;
            c.aux = (j < S.pend_n) ? 1 : 0;
            ctx_meta[r] = c;
        }
    }
}

template <typename T>
void launch_embed_norm(const T *emb, int H, SeqState *st, const int *active, int nseq, int B, int is_draft,
                       const int *drafts, int mask_id, float *x, RowMeta *meta, RowMeta *ctx_meta, const float *g, T *xg,
                       int xg_ld, size_t lo, float *ssq, int ssq_ld, cudaStream_t s) {
    launch_k(embed_norm_kernel<T>, dim3(nseq * B), dim3(256), 0, s, 1, emb, H, st, active, B, is_draft, drafts, mask_id, x,
             meta, ctx_meta, g, xg, xg_ld, lo, ssq, ssq_ld);
}

template <typename T>
__global__ void embed_tokens_kernel(const T *__restrict__ emb, int H, const int *__restrict__ tokens,
                                    int seq, int pos0, float *__restrict__ x, RowMeta *meta) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int tok = tokens[r];
    copy_embedding_row(emb + (size_t)tok * H, x + (size_t)r * H, H);
    if (threadIdx.x == 0) {
        RowMeta m;
        m.seq = seq;
        m.pos = pos0 + r;
        m.nk = pos0 + r + 1;  // causal
        m.aux = r;            // prefill tap rows are chunk rows
        meta[r] = m;
    }
}

template <typename T>
void launch_embed_tokens(const T *emb, int H, const int *tokens, int R, int seq, int pos0, float *x,
                         RowMeta *meta, cudaStream_t s) {
    launch_k(embed_tokens_kernel<T>, dim3(R), dim3(256), 0, s, 1, emb, H, tokens, seq, pos0, x, meta);
}

__global__ void ctx_meta_prefill_kernel(RowMeta *meta, int R, int seq, int pos0) {
    pdl_trigger();
    pdl_wait();
    int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    RowMeta m;
    m.seq = seq;
    m.pos = pos0 + r;
    m.nk = 0;
    m.aux = 1;
    meta[r] = m;
}

void launch_ctx_meta_prefill(RowMeta *meta, int R, int seq, int pos0, cudaStream_t s) {
    launch_k(ctx_meta_prefill_kernel, dim3((R + 127) / 128), dim3(128), 0, s, 1, meta, R, seq, pos0);
}

// ------------------------------------------------------------------------
// RMSNorm: out = x / sqrt(mean(x^2) + eps) * g   (fp32 statistics)
// ------------------------------------------------------------------------

template <typename TO>
__global__ void rmsnorm_kernel(const float *__restrict__ x, int ldx, const float *__restrict__ g,
                               int H, float eps, TO *__restrict__ out, int ldo, size_t lo) {
    pdl_trigger();
    pdl_wait();
    // the row is held in registers (float4 chunks, all loads issued before any
    // use); rows longer than NV * 4 * blockDim columns are re-read in a tail loop
    constexpr int NV = 8;
    const int r = blockIdx.x;
    const float4 *x4 = reinterpret_cast<const float4 *>(x + (size_t)r * ldx);
    const float4 *g4 = reinterpret_cast<const float4 *>(g);
    const int H4 = H >> 2;
    float4 v[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int c = threadIdx.x + u * blockDim.x;
        v[u] = c < H4 ? x4[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < NV; ++u) ss += (v[u].x * v[u].x + v[u].y * v[u].y) + (v[u].z * v[u].z + v[u].w * v[u].w);
    for (int c = threadIdx.x + NV * blockDim.x; c < H4; c += blockDim.x) {
        const float4 t = x4[c];
        ss += (t.x * t.x + t.y * t.y) + (t.z * t.z + t.w * t.w);
    }
    __shared__ float red[32];
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float w = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        w = warp_sum(w);
        if (threadIdx.x == 0) red[0] = w;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] / (float)H + eps);
    const size_t o0 = (size_t)r * ldo;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int c = threadIdx.x + u * blockDim.x;
        if (c < H4) {
            const float4 gg = g4[c];
            st_act(out, o0 + 4 * c + 0, lo, v[u].x * inv * gg.x);
            st_act(out, o0 + 4 * c + 1, lo, v[u].y * inv * gg.y);
            st_act(out, o0 + 4 * c + 2, lo, v[u].z * inv * gg.z);
            st_act(out, o0 + 4 * c + 3, lo, v[u].w * inv * gg.w);
        }
    }
    for (int c = threadIdx.x + NV * blockDim.x; c < H4; c += blockDim.x) {
        const float4 t = x4[c], gg = g4[c];
        st_act(out, o0 + 4 * c + 0, lo, t.x * inv * gg.x);
        st_act(out, o0 + 4 * c + 1, lo, t.y * inv * gg.y);
        st_act(out, o0 + 4 * c + 2, lo, t.z * inv * gg.z);
        st_act(out, o0 + 4 * c + 3, lo, t.w * inv * gg.w);
    }
}

template <typename TO>
void launch_rmsnorm(const float *x, int ldx, const float *g, int H, float eps, TO *out, int ldo, size_t lo, int R,
                    cudaStream_t s) {
    if (R <= 0) return;
    launch_k(rmsnorm_kernel<TO>, dim3(R), dim3(256), 0, s, 1, x, ldx, g, H, eps, out, ldo, lo);
}

// ------------------------------------------------------------------------
// residual add (+ tap copies), SwiGLU, QKV RoPE + KV write
// ------------------------------------------------------------------------

template <typename T>
__global__ void residual_kernel(float *__restrict__ x, const float *__restrict__ Y, int ldy, int H,
                                TapDst<T> taps, size_t lo, const RowMeta *__restrict__ meta) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    float *xr = x + (size_t)r * H;
    const float *yr = Y + (size_t)r * ldy;
    const int trow = taps.n ? meta[r].aux : 0;
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        float v = xr[c] + yr[c];
        xr[c] = v;
        for (int t = 0; t < taps.n; ++t)
            st_act(taps.base, (size_t)trow * taps.ld + taps.col[t] + c, lo, v);
    }
}

template <typename T>
void launch_residual(float *x, const float *Y, int ldy, int H, int R, const TapDst<T> &taps, size_t lo,
                     const RowMeta *meta, cudaStream_t s) {
    if (R <= 0) return;
    launch_k(residual_kernel<T>, dim3(R), dim3(256), 0, s, 1, x, Y, ldy, H, taps, lo, meta);
}

template <typename T>
__global__ void swiglu_kernel(const float *__restrict__ Y, int ldy, int F, T *__restrict__ h, int ldh, size_t lo) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= F) return;
    const float gt = Y[(size_t)r * ldy + c], up = Y[(size_t)r * ldy + F + c];
    st_act(h, (size_t)r * ldh + c, lo, silu_f(gt) * up);
}

template <typename T>
void launch_swiglu(const float *Y, int ldy, int F, int R, T *h, int ldh, size_t lo, cudaStream_t s) {
    if (R <= 0) return;
    dim3 grid((F + 255) / 256, R);
    launch_k(swiglu_kernel<T>, dim3(grid), dim3(256), 0, s, 1, Y, ldy, F, h, ldh, lo);
}

// Y columns c correspond to rows col0 + c of the layer's Wqkv = [Wq; Wk; Wv].
// Block rows (r < R_blk): q -> RoPE -> q_out; k -> RoPE -> kc; v -> vc at meta.pos.
// Context rows (r >= R_blk): k -> RoPE -> kc; v -> vc at ctx_meta.pos when ctx_meta.aux.
template <typename T>
__global__ void qkv_epilogue_kernel(const float *__restrict__ Y, int ldy, int col0, int R_blk,
                                    const RowMeta *__restrict__ meta, const RowMeta *__restrict__ ctx_meta,
                                    int nq, int nkv, int hd, const float2 *__restrict__ rope,
                                    T *__restrict__ q_out, T *__restrict__ kc, T *__restrict__ vc,
                                    int max_len, size_t lo, const float *__restrict__ qn_g,
                                    const float *__restrict__ kn_g, float qk_eps) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const bool is_ctx = r >= R_blk;
    RowMeta m = is_ctx ? ctx_meta[r - R_blk] : meta[r];
    if (is_ctx && !m.aux) return;
    const int qd = nq * hd, kd = nkv * hd, half = hd / 2;
    const float *y = Y + (size_t)r * ldy - col0;   // y[c] for global Wqkv row c
    const float2 *tab = rope + (size_t)m.pos * half;
    const int c_begin = is_ctx ? qd : 0;
    // QK-norm: 1 / rms of every q and k head of this row (one warp per head)
    __shared__ float hs[256];  // nq + nkv <= 256 (checked at create)
    if (qn_g) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int head = warp; head < nq + nkv; head += blockDim.x >> 5) {
            float a = 0.f;
            if (!(head < nq && is_ctx))
                for (int d = lane; d < hd; d += 32) a += y[head * hd + d] * y[head * hd + d];
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (lane == 0) hs[head] = 1.0f / sqrtf(a / (float)hd + qk_eps);
        }
        __syncthreads();
    }
    // RoPE pairs over q and k heads
    for (int e = threadIdx.x; e < (nq + nkv) * half; e += blockDim.x) {
        const int head = e / half, i = e % half;
        if (head < nq && is_ctx) continue;
        const int base = head * hd;  // q heads then k heads (k starts at qd)
        float x1 = y[base + i], x2 = y[base + i + half];
        if (qn_g) {
            const float *g = head < nq ? qn_g : kn_g;
            x1 *= hs[head] * g[i];
            x2 *= hs[head] * g[i + half];
        }
        const float2 cs = tab[i];
        const float o1 = x1 * cs.x - x2 * cs.y, o2 = x2 * cs.x + x1 * cs.y;
        if (head < nq) {
            st_act(q_out, (size_t)r * qd + base + i, lo, o1);
            st_act(q_out, (size_t)r * qd + base + i + half, lo, o2);
        } else {
            const int kh = head - nq;
            T *dst = kc + (((size_t)m.seq * nkv + kh) * max_len + m.pos) * hd;
            st_act(dst, i, lo, o1);
            st_act(dst, i + half, lo, o2);
        }
    }
    (void)c_begin;
    for (int e = threadIdx.x; e < kd; e += blockDim.x) {
        const int kh = e / hd, d = e % hd;
        T *dst = vc + (((size_t)m.seq * nkv + kh) * max_len + m.pos) * hd;
        st_act(dst, d, lo, y[qd + kd + e]);
    }
}

template <typename T>
void launch_qkv_epilogue(const float *Y, int ldy, int col0, int R_blk, int R_tot, const RowMeta *meta,
                         const RowMeta *ctx_meta, int nq, int nkv, int hd, const float2 *rope, T *q_out,
                         T *kc, T *vc, int max_len, size_t lo, const float *qn_g, const float *kn_g, float qk_eps,
                         cudaStream_t s) {
    if (R_tot <= 0) return;
    launch_k(qkv_epilogue_kernel<T>, dim3(R_tot), dim3(128), 0, s, 1, Y, ldy, col0, R_blk, meta, ctx_meta, nq, nkv, hd, rope,
                                                 q_out, kc, vc, max_len, lo, qn_g, kn_g, qk_eps);
}

// ------------------------------------------------------------------------
// greedy heads
// ------------------------------------------------------------------------

__global__ void argmax_rows_kernel(const float *__restrict__ logits, int64_t ldl, int V, int mode, int B,
                                   int *__restrict__ idx, DevStats *stats) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    if (mode == 1 && (r % B) == 0) return;
    const float *l = logits + (size_t)r * ldl;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    bool bad = false;
    for (int c = threadIdx.x; c < V; c += blockDim.x) {
        float v = l[c];
        if (!isfinite(v)) bad = true;
        argmax_merge(best, bi, v, c);
    }
    __shared__ float sv[32];
    __shared__ int si[32];
    for (int o = 16; o > 0; o >>= 1) {
        float v2 = __shfl_xor_sync(0xffffffffu, best, o);
        int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        argmax_merge(best, bi, v2, i2);
    }
    if ((threadIdx.x & 31) == 0) { sv[threadIdx.x >> 5] = best; si[threadIdx.x >> 5] = bi; }
    if (bad && stats) atomicOr(&stats->status, 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        best = sv[0];
        bi = si[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) argmax_merge(best, bi, sv[w], si[w]);
        if (bi >= V) bi = 0;
        if (mode == 0) idx[r] = bi;
        else idx[(r / B) * (B - 1) + (r % B) - 1] = bi;
    }
}

void launch_argmax_rows(const float *logits, int64_t ldl, int V, int R, int mode, int B, int *idx,
                        DevStats *stats, cudaStream_t s) {
    if (R <= 0) return;
    launch_k(argmax_rows_kernel, dim3(R), dim3(512), 0, s, 1, logits, ldl, V, mode, B, idx, stats);
}

// ------------------------------------------------------------------------
// accept + commit (greedy, lossless) and token scripts
// ------------------------------------------------------------------------

__global__ void accept_kernel(SeqState *st, const int *__restrict__ active, int nseq, int B,
                              const int *__restrict__ drafts, const int *__restrict__ g, int *accept,
                              int *committed, int *new_len, int *out_tok, int out_ld, DevStats *stats) {
    pdl_trigger();
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int s = active[i];
    SeqState S = st[s];
    const int *d = drafts + i * (B - 1);
    const int *gi = g + i * B;
    int a = 0;
    if (!S.done)
        while (a < B - 1 && d[a] == gi[a]) ++a;
    const bool live = !S.done;
    commit_block(S, s, i, a, d, gi[a], B, committed, out_tok, out_ld, stats);
    if (live) st[s] = S;
    if (accept) accept[i] = a;
    if (new_len) new_len[i] = S.len;
}

void launch_accept(SeqState *st, const int *active, int nseq, int B, const int *drafts, const int *g,
                   int *accept, int *committed, int *new_len, int *out_tok, int out_ld, DevStats *stats,
                   cudaStream_t s) {
    launch_k(accept_kernel, dim3((nseq + 127) / 128), dim3(128), 0, s, 1, st, active, nseq, B, drafts, g, accept, committed,
                                                     new_len, out_tok, out_ld, stats);
}

__global__ void script_drafts_kernel(const SeqState *st, const int *__restrict__ active, int nseq, int B,
                                     int tau, int V, const int *__restrict__ script, int script_ld,
                                     int *drafts) {
    pdl_trigger();
    pdl_wait();
    const int i = blockIdx.x;
    const int k = threadIdx.x;
    if (i >= nseq || k >= B - 1) return;
    const int s = active[i];
    int idx = st[s].n_out + k;
    if (idx >= script_ld) idx = script_ld - 1;
    int tok = script[(size_t)s * script_ld + idx];
    if (k == tau - 1) tok = (tok + 1) % V;
    drafts[i * (B - 1) + k] = tok;
}

void launch_script_drafts(const SeqState *st, const int *active, int nseq, int B, int tau, int V,
                          const int *script, int script_ld, int *drafts, cudaStream_t s) {
    if (B <= 1 || nseq <= 0) return;
    launch_k(script_drafts_kernel, dim3(nseq), dim3(32 * ((B + 30) / 32)), 0, s, 1, st, active, nseq, B, tau, V, script,
                                                               script_ld, drafts);
}

__global__ void prefill_finish_kernel(SeqState *st, int seq, int n, const int *first_tok, int *out_tok,
                                      int out_ld, int max_new) {
    pdl_trigger();
    pdl_wait();
    SeqState S;
    S.len = n;
    S.anchor = *first_tok;
    S.ctx_len = n;
    S.pend_pos0 = n;
    S.pend_n = 0;
    S.n_out = max_new > 0 ? 1 : 0;
    S.max_new = max_new;
    S.done = max_new <= 1 ? 1 : 0;
    if (max_new > 0) out_tok[(size_t)seq * out_ld] = S.anchor;
    st[seq] = S;
}

void launch_prefill_finish(SeqState *st, int seq, int n, const int *first_tok, int *out_tok, int out_ld,
                           int max_new, cudaStream_t s) {
    launch_k(prefill_finish_kernel, dim3(1), dim3(1), 0, s, 1, st, seq, n, first_tok, out_tok, out_ld, max_new);
}

// target-only greedy step: g is the argmax of the single row of each sequence
__global__ void ar_step_kernel(SeqState *st, const int *__restrict__ active, int nseq, const int *g,
                               int *out_tok, int out_ld, DevStats *stats) {
    pdl_trigger();
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int s = active[i];
    SeqState S = st[s];
    if (S.done) return;
    const int tok = g[i];
    out_tok[(size_t)s * out_ld + S.n_out] = tok;
    S.n_out++;
    S.anchor = tok;
    if (S.n_out >= S.max_new) {
        S.done = 1;
        if (stats) atomicAdd(&stats->n_done, 1);
    } else {
        S.len += 1;
    }
    st[s] = S;
}

void launch_ar_step(SeqState *st, const int *active, int nseq, const int *g, int *out_tok, int out_ld,
                    DevStats *stats, cudaStream_t s) {
    launch_k(ar_step_kernel, dim3((nseq + 127) / 128), dim3(128), 0, s, 1, st, active, nseq, g, out_tok, out_ld, stats);
}

// ------------------------------------------------------------------------
// RoPE table: (cos, sin)(pos * theta^(-2i/hd)), angles in double precision
// ------------------------------------------------------------------------

// RoPE frequency of pair i; factor > 1: Llama 3.1 rescaling by wavelength band
__device__ double rope_freq(int i, int hd, double theta, double factor, double low, double high, double orig) {
    const double f = pow(theta, -2.0 * (double)i / (double)hd);
    if (!(factor > 1.0)) return f;
    const double wavelen = 2.0 * 3.14159265358979323846 / f;
    if (wavelen < orig / high) return f;        // short wavelengths: kept
    if (wavelen > orig / low) return f / factor;  // long wavelengths: divided by the factor
    const double sm = (orig / wavelen - low) / (high - low);
    return (1.0 - sm) * f / factor + sm * f;
}

__global__ void rope_table_kernel(float2 *tab, int max_len, int hd, double theta, double factor, double low,
                                  double high, double orig) {
    pdl_trigger();
    pdl_wait();
    const int half = hd / 2;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)max_len * half) return;
    const int pos = (int)(e / half), i = (int)(e % half);
    const double freq = rope_freq(i, hd, theta, factor, low, high, orig);
    double sn, cs;
    sincos((double)pos * freq, &sn, &cs);
    tab[e] = make_float2((float)cs, (float)sn);
}

void launch_rope_table(float2 *tab, int max_len, int hd, double theta, double factor, double low, double high,
                       double orig, cudaStream_t s) {
    const int64_t n = (int64_t)max_len * (hd / 2);
    launch_k(rope_table_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, 1, tab, max_len, hd, theta,
             factor, low, high, orig);
}

// ------------------------------------------------------------------------
// explicit instantiations
// ------------------------------------------------------------------------
#define DFL_INST(T)                                                                                         \
    template void launch_embed_norm<T>(const T *, int, SeqState *, const int *, int, int, int, const int *, int, \
                                       float *, RowMeta *, RowMeta *, const float *, T *, int, size_t, float *, int, \
                                       cudaStream_t);                                                           \
    template void launch_embed_block<T>(const T *, int, SeqState *, const int *, int, int, int, const int *, \
                                        int, float *, RowMeta *, RowMeta *, cudaStream_t);                  \
    template void launch_embed_tokens<T>(const T *, int, const int *, int, int, int, float *, RowMeta *,    \
                                         cudaStream_t);                                                     \
    template void launch_rmsnorm<T>(const float *, int, const float *, int, float, T *, int, size_t, int,   \
                                    cudaStream_t);                                                          \
    template void launch_residual<T>(float *, const float *, int, int, int, const TapDst<T> &, size_t,      \
                                     const RowMeta *, cudaStream_t);                                        \
    template void launch_swiglu<T>(const float *, int, int, int, T *, int, size_t, cudaStream_t);           \
    template void launch_qkv_epilogue<T>(const float *, int, int, int, int, const RowMeta *,                \
                                         const RowMeta *, int, int, int, const float2 *, T *, T *, T *,     \
                                         int, size_t, const float *, const float *, float, cudaStream_t);
DFL_INST(float)
DFL_INST(bf16)
#undef DFL_INST

}  // namespace dfl

namespace dfl {

// dst rows i*B + j  <-  src rows active[i]*B + j  (16-byte words)
__global__ void gather_rows_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, size_t row_words,
                                   const int *__restrict__ active, int B) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int i = r / B, j = r % B;
    const uint4 *s = src + ((size_t)active[i] * B + j) * row_words;
    uint4 *d = dst + (size_t)r * row_words;
    for (size_t w = threadIdx.x; w < row_words; w += blockDim.x) d[w] = s[w];
}

void launch_gather_rows(const void *src, void *dst, size_t row_bytes, const int *active, int nseq, int B,
                        cudaStream_t s) {
    if (nseq <= 0) return;
    launch_k(gather_rows_kernel, dim3(nseq * B), dim3(256), 0, s, 1, (const uint4 *)src, (uint4 *)dst, row_bytes / 16, active, B);
}

}  // namespace dfl
