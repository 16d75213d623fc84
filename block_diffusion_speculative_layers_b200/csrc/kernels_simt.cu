// kernels_simt.cu -- CUDA-core kernels for fp32 models (the tiny correctness
// configuration computes in fp32 end to end, where tensor-core bf16 inputs
// would change the model): GEMM, attention and MoE experts, plus the MoE
// combine every dtype uses.  bf16 models use the tensor-core kernels in
// gemm_tc.cu and attn_mma.cu and the expert kernels in moe_experts.cu instead.
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
