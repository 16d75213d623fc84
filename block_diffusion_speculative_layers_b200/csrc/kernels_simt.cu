// kernels_simt.cu -- CUDA-core kernels for fp32 models (the tiny correctness
// configuration computes in fp32 end to end, where tensor-core bf16 inputs
// would change the model): GEMM, attention and MoE experts.  bf16 models use
// the tensor-core kernels in gemm_tc.cu and attn_mma.cu instead.
#include <math.h>

#include "kernels.h"
#include "launch.h"

namespace dfl {

// ------------------------------------------------------------------------
// GEMM: Y[M][N] = X[M][K] . W[N][K]^T, fp32 accumulate
// ------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T *__restrict__ X, int ldx, int M,
                                                        const T *__restrict__ W, int ldw, int N, int K,
                                                        float *__restrict__ Y, int ldy, size_t lo) {
    pdl_trigger();
    pdl_wait();
    __shared__ float Ws[64][33];
    __shared__ float Xs[32][33];
    const int n0 = blockIdx.x * 64, m0 = blockIdx.y * 32;
    const int tid = threadIdx.x, tx = tid & 63, ty = tid >> 6;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            const int n = n0 + rr, k = k0 + kk;
            Ws[rr][kk] = (n < N && k < K) ? to_f(W[(size_t)n * ldw + k]) : 0.f;
        }
        for (int e = tid; e < 32 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            const int m = m0 + rr, k = k0 + kk;
            Xs[rr][kk] = (m < M && k < K) ? ld_act(X, (size_t)m * ldx + k, lo) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            const float w = Ws[tx][kk];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(Xs[ty * 8 + i][kk], w, acc[i]);
        }
        __syncthreads();
    }
    const int n = n0 + tx;
    if (n < N)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = m0 + ty * 8 + i;
            if (m < M) Y[(size_t)m * ldy + n] = acc[i];
        }
}

template <typename T>
void launch_gemm_simt(const T *X, int ldx, int M, const T *W, int ldw, int N, int K, float *Y, int ldy,
                      size_t lo, cudaStream_t s) {
    if (M <= 0 || N <= 0) return;
    dim3 grid((N + 63) / 64, (M + 31) / 32);
    launch_k(gemm_simt_kernel<T>, dim3(grid), dim3(256), 0, s, 1, X, ldx, M, W, ldw, N, K, Y, ldy, lo);
}

// ------------------------------------------------------------------------
// attention: one warp per (row, q head); online softmax over visible keys
// [0, meta.nk) of the row's sequence; q head h reads kv head h / (nq/nkv).
// ------------------------------------------------------------------------
template <typename T>
__global__ void attention_simt_kernel(const T *__restrict__ q, int ldq, const T *__restrict__ kc,
                                      const T *__restrict__ vc, const RowMeta *__restrict__ meta, int nq,
                                      int nkv, int hd, int max_len, float scale, T *__restrict__ out,
                                      int ldo) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
    const RowMeta m = meta[r];
    const int kvh = h / (nq / nkv);
    const size_t base = ((size_t)m.seq * nkv + kvh) * (size_t)max_len * hd;
    const T *K = kc + base;
    const T *V = vc + base;
    const int per = hd / 32;
    float qv[8], acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        qv[i] = i < per ? to_f(q[(size_t)r * ldq + h * hd + lane + 32 * i]) : 0.f;
        acc[i] = 0.f;
    }
    float mx = -INFINITY, den = 0.f;
    for (int j = 0; j < m.nk; ++j) {
        float sc = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < per) sc += qv[i] * to_f(K[(size_t)j * hd + lane + 32 * i]);
        sc = warp_sum(sc) * scale;
        const float mn = fmaxf(mx, sc);
        const float corr = expf(mx - mn);
        const float p = expf(sc - mn);
        den = den * corr + p;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < per) acc[i] = acc[i] * corr + p * to_f(V[(size_t)j * hd + lane + 32 * i]);
        mx = mn;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < per) out[(size_t)r * ldo + h * hd + lane + 32 * i] = from_f<T>(acc[i] / den);
}

template <typename T>
void launch_attention_simt(const T *q, int ldq, const T *kc, const T *vc, const RowMeta *meta, int R, int nq,
                           int nkv, int hd, int max_len, T *out, int ldo, cudaStream_t s) {
    if (R <= 0) return;
    dim3 grid(R, nq);
    launch_k(attention_simt_kernel<T>, dim3(grid), dim3(32), 0, s, 1, q, ldq, kc, vc, meta, nq, nkv, hd, max_len,
                                                 1.0f / sqrtf((float)hd), out, ldo);
}

// ------------------------------------------------------------------------
// MoE routing: softmax over experts, top-k (lowest index on ties),
// weights renormalised over the chosen k.  One warp per row.
// ------------------------------------------------------------------------
__global__ void moe_topk_kernel(const float *__restrict__ lg, int E, int R, int k, int *sel, float *wt) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= R) return;
    const float *l = lg + (size_t)r * E;
    float mx = -INFINITY;
    for (int e = lane; e < E; e += 32) mx = fmaxf(mx, l[e]);
    mx = warp_max(mx);
    unsigned used[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // E <= 256
    float psum = 0.f;
    float chosen_p[32];
    int chosen_e[32];
    for (int t = 0; t < k; ++t) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            if ((used[e >> 5] >> (e & 31)) & 1u) continue;
            argmax_merge(bv, bi, l[e], e);
        }
        for (int o = 16; o > 0; o >>= 1) {
            float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
            int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
            argmax_merge(bv, bi, v2, i2);
        }
        used[bi >> 5] |= 1u << (bi & 31);
        const float p = expf(bv - mx);
        chosen_p[t] = p;
        chosen_e[t] = bi;
        psum += p;
    }
    if (lane == 0)
        for (int t = 0; t < k; ++t) {
            sel[r * k + t] = chosen_e[t];
            wt[r * k + t] = chosen_p[t] / psum;
        }
}

void launch_moe_topk(const float *router_logits, int E, int R, int k, int *sel, float *wt, cudaStream_t s) {
    if (R <= 0) return;
    launch_k(moe_topk_kernel, dim3((R + 3) / 4), dim3(128), 0, s, 1, router_logits, E, R, k, sel, wt);
}

// Expert FFN per (row, choice): part[rk] = W_down_e (SiLU(W_gate_e m) * W_up_e m)
template <typename T>
__global__ void moe_experts_simt_kernel(const T *__restrict__ m, int ldm, size_t lo, int k, const int *__restrict__ sel,
                                        const T *__restrict__ w_gate_up, const T *__restrict__ w_down, int H,
                                        int Fe, float *__restrict__ part) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float sm[];
    float *xs = sm;          // [H]
    float *gu = sm + H;      // [2Fe]
    const int rk = blockIdx.x, r = rk / k;
    const int e = sel[rk];
    for (int c = threadIdx.x; c < H; c += blockDim.x) xs[c] = ld_act(m, (size_t)r * ldm + c, lo);
    __syncthreads();
    const T *Wgu = w_gate_up + (size_t)e * 2 * Fe * H;
    for (int o = threadIdx.x; o < 2 * Fe; o += blockDim.x) {
        const T *w = Wgu + (size_t)o * H;
        float a = 0.f;
        for (int c = 0; c < H; ++c) a = fmaf(to_f(w[c]), xs[c], a);
        gu[o] = a;
    }
    __syncthreads();
    // the expert's hidden activation is a GEMM input: rounded like a stored one
    // (single bf16 plane), or kept at fp32 where two planes would carry it
    for (int i = threadIdx.x; i < Fe; i += blockDim.x) {
        const float hv = silu_f(gu[i]) * gu[Fe + i];
        gu[i] = lo ? hv : to_f(from_f<T>(hv));
    }
    __syncthreads();
    const T *Wd = w_down + (size_t)e * H * Fe;
    for (int o = threadIdx.x; o < H; o += blockDim.x) {
        const T *w = Wd + (size_t)o * Fe;
        float a = 0.f;
        for (int c = 0; c < Fe; ++c) a = fmaf(to_f(w[c]), gu[c], a);
        part[(size_t)rk * H + o] = a;
    }
}

template <typename T>
void launch_moe_experts_simt(const T *m, int ldm, size_t lo, int R, int k, const int *sel, const T *w_gate_up,
                             const T *w_down, int H, int Fe, float *part, cudaStream_t s) {
    if (R <= 0) return;
    const size_t smem = sizeof(float) * (size_t)(H + 2 * Fe);
    launch_k(moe_experts_simt_kernel<T>, dim3(R * k), dim3(256), smem, s, 1, m, ldm, lo, k, sel, w_gate_up, w_down, H, Fe,
             part);
}

// ------------------------------------------------------------------------
// MoE experts, bucketed: every (row, choice) pair is listed under its expert,
// then one CTA group per touched expert streams that expert's weights exactly
// once (warp per weight row, 16-byte coalesced loads) and applies them to all
// of the expert's rows staged in shared memory.  Experts no row routes to are
// not read at all.
// ------------------------------------------------------------------------
constexpr int MOE_PC = 4;  // expert rows staged per pass

// pairs rk = r*k + t grouped by expert: off[e] .. off[e+1]-1 index list[]
__global__ void moe_bucket_kernel(const int *__restrict__ sel, int n_pairs, int E, int *off, int *list) {
    pdl_trigger();
    pdl_wait();
    __shared__ int cnt[257], cur[256];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n_pairs; i += blockDim.x) atomicAdd(&cnt[sel[i]], 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            const int c = cnt[e];
            cnt[e] = acc;
            cur[e] = acc;
            acc += c;
        }
        cnt[E] = acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) off[e] = cnt[e];
    // the order of pairs within an expert does not matter: each pair has its own output row
    for (int i = threadIdx.x; i < n_pairs; i += blockDim.x) list[atomicAdd(&cur[sel[i]], 1)] = i;
}

__device__ __forceinline__ void bf16x8_to_f(const uint4 &u, float *f) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(b[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

constexpr int MOE_CPL = 12;  // 16-byte weight chunks per lane and row (rows of up to 3072 bf16)

// x rows of pairs c0 .. c0+nc-1 of the expert into xs[j][0..n) (fp32, both planes summed):
// 16-byte loads of every staged row issued before any is used (n % 8 == 0, rows 16-byte aligned)
template <typename T>
__device__ __forceinline__ void moe_stage(const T *__restrict__ src, int ld, size_t lo, const int *__restrict__ list,
                                          int p0, int c0, int nc, int div, int n, float *xs) {
    int row[MOE_PC];
#pragma unroll
    for (int j = 0; j < MOE_PC; ++j) row[j] = j < nc ? list[p0 + c0 + j] / div : 0;
    for (int c = threadIdx.x; c < n / 8; c += blockDim.x) {
        uint4 hi[MOE_PC], lw[MOE_PC];
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) {
            if (j >= nc) break;
            const size_t at = (size_t)row[j] * ld + (size_t)c * 8;
            hi[j] = *reinterpret_cast<const uint4 *>(src + at);
            if (lo) lw[j] = *reinterpret_cast<const uint4 *>(src + lo + at);
        }
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) {
            if (j >= nc) break;
            float a[8], b[8];
            bf16x8_to_f(hi[j], a);
            if (lo) bf16x8_to_f(lw[j], b);
#pragma unroll
            for (int t = 0; t < 8; ++t) xs[j * n + c * 8 + t] = lo ? a[t] + b[t] : a[t];
        }
    }
}

// dot products of one weight row (in registers: lane's chunks q*32 + lane) with nc staged rows
__device__ __forceinline__ void moe_dots(const uint4 *wr, int cpl, const float *xs, int n, int nc, float *acc) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < MOE_CPL; ++q) {
        if (q >= cpl) break;
        float a[8];
        bf16x8_to_f(wr[q], a);
        const int col = (q * 32 + lane) * 8;
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) {
            if (j >= nc) break;
            const float4 x0 = *reinterpret_cast<const float4 *>(xs + j * n + col);
            const float4 x1 = *reinterpret_cast<const float4 *>(xs + j * n + col + 4);
            acc[j] += a[0] * x0.x + a[1] * x0.y + a[2] * x0.z + a[3] * x0.w + a[4] * x1.x + a[5] * x1.y + a[6] * x1.z +
                      a[7] * x1.w;
        }
    }
}

// gate/up of expert blockIdx.x, one warp per column f = blockIdx.y * 8 + warp:
// h[pair][f] = SiLU(W_gate[f] . m[row]) * (W_up[f] . m[row]) for every pair of the expert.
// Both weight rows are loaded before the expert's rows are staged.  H % 256 == 0.
template <typename T>
__global__ void __launch_bounds__(256) moe_gateup_kernel(const T *__restrict__ m, int ldm, size_t lo, int k,
                                                         const int *__restrict__ off, const int *__restrict__ list,
                                                         const T *__restrict__ w_gate_up, int H, int Fe,
                                                         T *__restrict__ h, size_t hlo) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float xs[];  // [MOE_PC][H]
    const int e = blockIdx.x;
    const int p0 = off[e], np = off[e + 1] - p0;
    if (np == 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f = blockIdx.y * 8 + warp;
    const int cpl = H / 256;
    uint4 wg[MOE_CPL], wu[MOE_CPL];
    if (f < Fe) {
        const uint4 *g = reinterpret_cast<const uint4 *>(w_gate_up + ((size_t)e * 2 * Fe + f) * H);
        const uint4 *u = reinterpret_cast<const uint4 *>(w_gate_up + ((size_t)e * 2 * Fe + Fe + f) * H);
#pragma unroll
        for (int q = 0; q < MOE_CPL; ++q)
            if (q < cpl) {
                wg[q] = __ldg(g + q * 32 + lane);
                wu[q] = __ldg(u + q * 32 + lane);
            }
    }
    for (int c0 = 0; c0 < np; c0 += MOE_PC) {
        const int nc = min(MOE_PC, np - c0);
        __syncthreads();
        moe_stage(m, ldm, lo, list, p0, c0, nc, k, H, xs);
        __syncthreads();
        if (f >= Fe) continue;
        float gs[MOE_PC], us[MOE_PC];
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) gs[j] = us[j] = 0.f;
        moe_dots(wg, cpl, xs, H, nc, gs);
        moe_dots(wu, cpl, xs, H, nc, us);
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) {
            const float a = warp_sum(gs[j]), b = warp_sum(us[j]);
            if (lane == 0 && j < nc) st_act(h, (size_t)list[p0 + c0 + j] * Fe + f, hlo, silu_f(a) * b);
        }
    }
}

// down of expert blockIdx.x, one warp per output o = blockIdx.y * 8 + warp:
// part[pair][o] = W_down[o] . h[pair].  Fe % 256 == 0.
template <typename T>
__global__ void __launch_bounds__(256) moe_down_kernel(const T *__restrict__ h, size_t hlo, const int *__restrict__ off,
                                                       const int *__restrict__ list, const T *__restrict__ w_down,
                                                       int H, int Fe, float *__restrict__ part) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float hs[];  // [MOE_PC][Fe]
    const int e = blockIdx.x;
    const int p0 = off[e], np = off[e + 1] - p0;
    if (np == 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int o = blockIdx.y * 8 + warp;
    const int cpl = Fe / 256;
    uint4 wr[MOE_CPL];
    if (o < H) {
        const uint4 *w = reinterpret_cast<const uint4 *>(w_down + ((size_t)e * H + o) * Fe);
#pragma unroll
        for (int q = 0; q < MOE_CPL; ++q)
            if (q < cpl) wr[q] = __ldg(w + q * 32 + lane);
    }
    for (int c0 = 0; c0 < np; c0 += MOE_PC) {
        const int nc = min(MOE_PC, np - c0);
        __syncthreads();
        moe_stage(h, Fe, hlo, list, p0, c0, nc, 1, Fe, hs);
        __syncthreads();
        if (o >= H) continue;
        float acc[MOE_PC];
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) acc[j] = 0.f;
        moe_dots(wr, cpl, hs, Fe, nc, acc);
#pragma unroll
        for (int j = 0; j < MOE_PC; ++j) {
            const float sum = warp_sum(acc[j]);
            if (lane == 0 && j < nc) part[(size_t)list[p0 + c0 + j] * H + o] = sum;
        }
    }
}

bool moe_bucketed_supported(int H, int Fe, int E) {
    return H % 256 == 0 && Fe % 256 == 0 && H <= 256 * MOE_CPL && Fe <= 256 * MOE_CPL && E <= 256;
}

void launch_moe_experts_bucketed(const bf16 *m, int ldm, size_t lo, int R, int k, const int *sel, int E,
                                 const bf16 *w_gate_up, const bf16 *w_down, int H, int Fe, int *off, int *list,
                                 bf16 *h, size_t hlo, float *part, cudaStream_t s) {
    if (R <= 0) return;
    launch_k(moe_bucket_kernel, dim3(1), dim3(1024), 0, s, 1, sel, R * k, E, off, list);
    launch_k(moe_gateup_kernel<bf16>, dim3(E, (Fe + 7) / 8), dim3(256), sizeof(float) * MOE_PC * H, s, 1, m, ldm, lo,
             k, (const int *)off, (const int *)list, w_gate_up, H, Fe, h, hlo);
    launch_k(moe_down_kernel<bf16>, dim3(E, (H + 7) / 8), dim3(256), sizeof(float) * MOE_PC * Fe, s, 1,
             (const bf16 *)h, hlo, (const int *)off, (const int *)list, w_down, H, Fe, part);
}

template <typename T>
__global__ void moe_combine_kernel(float *__restrict__ x, const float *__restrict__ part,
                                   const float *__restrict__ wt, int H, int k, TapDst<T> taps, size_t lo,
                                   const RowMeta *__restrict__ meta) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int trow = taps.n ? meta[r].aux : 0;
    // weighted sum over the k experts in selection order; the k partial rows of a
    // column group are loaded together (k <= 32, groups of 8)
    for (int c4 = threadIdx.x; c4 < H / 4; c4 += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int t0 = 0; t0 < k; t0 += 8) {
            float4 pv[8];
            float w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = t0 + u;
                w[u] = t < k ? wt[r * k + t] : 0.f;
                pv[u] = t < k ? reinterpret_cast<const float4 *>(part + ((size_t)r * k + t) * H)[c4]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x = fmaf(w[u], pv[u].x, acc.x);
                acc.y = fmaf(w[u], pv[u].y, acc.y);
                acc.z = fmaf(w[u], pv[u].z, acc.z);
                acc.w = fmaf(w[u], pv[u].w, acc.w);
            }
        }
        float4 *xr = reinterpret_cast<float4 *>(x + (size_t)r * H) + c4;
        float4 v = *xr;
        v.x += acc.x;
        v.y += acc.y;
        v.z += acc.z;
        v.w += acc.w;
        *xr = v;
        const float vv[4] = {v.x, v.y, v.z, v.w};
        for (int i = 0; i < taps.n; ++i)
            for (int u = 0; u < 4; ++u) st_act(taps.base, (size_t)trow * taps.ld + taps.col[i] + 4 * c4 + u, lo, vv[u]);
    }
}

template <typename T>
void launch_moe_combine(float *x, const float *part, const float *wt, int H, int R, int k,
                        const TapDst<T> &taps, size_t lo, const RowMeta *meta, cudaStream_t s) {
    if (R <= 0) return;
    launch_k(moe_combine_kernel<T>, dim3(R), dim3(256), 0, s, 1, x, part, wt, H, k, taps, lo, meta);
}

#define DFL_INST(T)                                                                                          \
    template void launch_gemm_simt<T>(const T *, int, int, const T *, int, int, int, float *, int, size_t,   \
                                      cudaStream_t);                                                         \
    template void launch_attention_simt<T>(const T *, int, const T *, const T *, const RowMeta *, int, int,  \
                                           int, int, int, T *, int, cudaStream_t);                           \
    template void launch_moe_experts_simt<T>(const T *, int, size_t, int, int, const int *, const T *, const T *, \
                                             int, int, float *, cudaStream_t);                               \
    template void launch_moe_combine<T>(float *, const float *, const float *, int, int, int,                \
                                        const TapDst<T> &, size_t, const RowMeta *, cudaStream_t);
DFL_INST(float)
DFL_INST(bf16)
#undef DFL_INST

}  // namespace dfl
