// sampling.cu -- temperature sampling of the draft-and-verify loop.
//
// With temperature T > 0 the LM heads store their fp32 logits rows and these
// kernels replace the greedy argmax and accept:
//   drafts   d_i ~ Q_i = softmax(z^draft_i / T)            (draw purpose DRAFT, position p + i)
//   accept   d_i while u * Q_i(d_i) < P_{i-1}(d_i),  P = softmax(z^verify / T)   (ACCEPT, p + i)
//   replace  the first rejected d_i by a draw from max(0, P_{i-1} - Q_i)       (RESIDUAL, p + i)
//   bonus    a draw from P_{B-1} when every draft is accepted                  (TARGET, p + B)
// which keeps the target's distribution (the standard speculative-sampling
// rule; greedy decoding is its T -> 0 limit).  Draws come from Philox4x32-10
// (philox.cuh) keyed by (seed, position, sequence slot, purpose); tokens are
// drawn by Gumbel-max, so every sampled token is an argmax of perturbed scores.
//
// sample_partials_kernel: CTA = (vocabulary chunk, row).  Per entry the scaled
// logit z/T feeds a running (max, sum of exp) and the perturbed score
// z/T + G(u) a running argmax; chunks are combined per row by
// sample_finish_kernel into the row's log-sum-exp and sampled token.
// residual_partials_kernel / residual_finish_kernel: the same over
// log(max(0, P - Q)) + G(u) for every block position of every sequence (only
// the first rejected one is used; computing all keeps the pass parallel).
// accept_sample_kernel: one thread per sequence applies the rule and commits.
#include <math.h>

#include "kernels.h"
#include "launch.h"
#include "philox.cuh"

namespace dfl {

namespace {

constexpr int CHUNK = 4096;  // vocabulary entries per CTA of the partial passes
constexpr int NT = 256;

__device__ __forceinline__ float gumbel_f(float u) { return -logf(-logf(u)); }

// running log-sum-exp state: m = max, s = sum of exp(z - m)
__device__ __forceinline__ void lse_add(float &m, float &s, float z) {
    if (z > m) {
        s = s * expf(m - z) + 1.f;
        m = z;
    } else {
        s += expf(z - m);
    }
}

__device__ __forceinline__ void lse_merge(float &m, float &s, float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        s = s2;
    } else if (m2 > m) {
        s = s * expf(m - m2) + s2;
        m = m2;
    } else {
        s += s2 * expf(m2 - m);
    }
}

// block-wide merge of (m, s, best value, best index) into thread 0
__device__ __forceinline__ void block_merge(float &m, float &s, float &bv, int &bi) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lse_merge(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
        argmax_merge(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
    }
    __shared__ float4 red[NT / 32];
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = make_float4(m, s, bv, __int_as_float(bi));
    __syncthreads();
    if (threadIdx.x == 0)
        for (int k = 1; k < NT / 32; ++k) {
            lse_merge(m, s, red[k].x, red[k].y);
            argmax_merge(bv, bi, red[k].z, __float_as_int(red[k].w));
        }
}

__global__ void __launch_bounds__(NT) sample_partials_kernel(SampleRows a) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.y, k = r % a.B;
    float4 *out = a.part + (size_t)blockIdx.x * a.R + r;
    if (a.mode == 1 && k == 0) return;
    const int slot = a.fixed_slot >= 0 ? a.fixed_slot : a.active[r / a.B];
    const uint32_t pos = (uint32_t)(a.fixed_pos >= 0 ? a.fixed_pos : a.st[slot].len + k + a.pos_off);
    const float *z = a.logits + (size_t)r * a.ldl;
    const int v0 = blockIdx.x * CHUNK, v1 = min(a.V, v0 + CHUNK);
    float m = -INFINITY, s = 0.f, bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int q = v0 / 4 + threadIdx.x; 4 * q < v1; q += NT) {
        float u[4];
        uniforms4(a.key, (uint32_t)q, pos, (uint32_t)slot, a.purpose, u);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int v = 4 * q + t;
            if (v < v1) {
                const float zs = z[v] * a.inv_T;
                lse_add(m, s, zs);
                argmax_merge(bv, bi, zs + gumbel_f(u[t]), v);
            }
        }
    }
    block_merge(m, s, bv, bi);
    if (threadIdx.x == 0) *out = make_float4(m, s, bv, __int_as_float(bi));
}

__global__ void sample_finish_kernel(SampleRows a, int n_chunks) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x, k = r % a.B, lane = threadIdx.x;
    if (a.mode == 1 && k == 0) return;
    float m = -INFINITY, s = 0.f, bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = lane; c < n_chunks; c += 32) {
        const float4 p = a.part[(size_t)c * a.R + r];
        lse_merge(m, s, p.x, p.y);
        argmax_merge(bv, bi, p.z, __float_as_int(p.w));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lse_merge(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
        argmax_merge(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
    }
    if (lane) return;
    if (!isfinite(m) || !isfinite(bv) || bi == 0x7fffffff) {
        if (a.stats) atomicOr(&a.stats->status, 1);
        bi = 0;
    }
    if (a.lse) a.lse[r] = m + logf(s);
    if (a.mode == 0)
        a.tok[r] = bi;
    else
        a.tok[(r / a.B) * (a.B - 1) + k - 1] = bi;
}

// row rr = i*(B-1) + k-1 (block position k = 1..B-1 of sequence i)
__global__ void __launch_bounds__(NT) residual_partials_kernel(ResidualRows a) {
    pdl_trigger();
    pdl_wait();
    const int rr = blockIdx.y, B = a.B, i = rr / (B - 1), k = rr % (B - 1) + 1;
    const int slot = a.active[i];
    const uint32_t pos = (uint32_t)(a.st[slot].len + k);
    const float *zp = a.plog + (size_t)(i * B + k - 1) * a.ldl;
    const float *zq = a.qlog + (size_t)(i * B + k) * a.ldl;
    const float lp = a.lse_p[i * B + k - 1], lq = a.lse_q[i * B + k];
    const int v0 = blockIdx.x * CHUNK, v1 = min(a.V, v0 + CHUNK);
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int q = v0 / 4 + threadIdx.x; 4 * q < v1; q += NT) {
        float u[4];
        uniforms4(a.key, (uint32_t)q, pos, (uint32_t)slot, SP_RESIDUAL, u);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int v = 4 * q + t;
            if (v < v1) {
                const float d = expf(zp[v] * a.inv_T - lp) - expf(zq[v] * a.inv_T - lq);
                if (d > 0.f) argmax_merge(bv, bi, logf(d) + gumbel_f(u[t]), v);
            }
        }
    }
    float m = -INFINITY, s = 0.f;
    block_merge(m, s, bv, bi);
    if (threadIdx.x == 0) a.part[(size_t)blockIdx.x * a.rows + rr] = make_float2(bv, __int_as_float(bi));
}

__global__ void residual_finish_kernel(ResidualRows a, int n_chunks) {
    pdl_trigger();
    pdl_wait();
    const int rr = blockIdx.x, lane = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = lane; c < n_chunks; c += 32) {
        const float2 p = a.part[(size_t)c * a.rows + rr];
        argmax_merge(bv, bi, p.x, __float_as_int(p.y));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        argmax_merge(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
    if (lane == 0) a.resid[rr] = bi == 0x7fffffff ? -1 : bi;  // -1: P <= Q everywhere (never rejected)
}

__global__ void accept_sample_kernel(AcceptSample a) {
    pdl_trigger();
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.nseq) return;
    const int s = a.active[i], B = a.B;
    SeqState S = a.st[s];
    const int *d = a.drafts + i * (B - 1);
    int acc = B - 1, x = a.tok_p[i * B + B - 1];  // bonus: the draw from P_{B-1}
    if (!S.done)
        for (int k = 1; k < B; ++k) {
            const int dk = d[k - 1];
            const float P = expf(a.plog[(size_t)(i * B + k - 1) * a.ldl + dk] * a.inv_T - a.lse_p[i * B + k - 1]);
            const float Q = expf(a.qlog[(size_t)(i * B + k) * a.ldl + dk] * a.inv_T - a.lse_q[i * B + k]);
            const float u = uniform1(a.key, (uint32_t)(S.len + k), (uint32_t)s, SP_ACCEPT);
            if (u * Q < P) continue;
            acc = k - 1;
            x = a.resid[i * (B - 1) + k - 1];
            if (x < 0) {  // a rejection leaves mass where P > Q; none means the logits were not finite
                if (a.stats) atomicOr(&a.stats->status, 1);
                x = 0;
            }
            break;
        }
    const bool live = !S.done;
    commit_block(S, s, i, acc, d, x, B, a.committed, a.out_tok, a.out_ld, a.stats);
    if (live) a.st[s] = S;
    if (a.accept) a.accept[i] = acc;
    if (a.new_len) a.new_len[i] = S.len;
}

}  // namespace

int sample_chunks(int V) { return (V + CHUNK - 1) / CHUNK; }

void launch_sample_rows(const SampleRows &a, cudaStream_t s) {
    if (a.R <= 0) return;
    const int nc = sample_chunks(a.V);
    launch_k(sample_partials_kernel, dim3(nc, a.R), dim3(NT), 0, s, 1, a);
    launch_k(sample_finish_kernel, dim3(a.R), dim3(32), 0, s, 1, a, nc);
}

void launch_residual_rows(const ResidualRows &a, cudaStream_t s) {
    if (a.rows <= 0) return;
    const int nc = sample_chunks(a.V);
    launch_k(residual_partials_kernel, dim3(nc, a.rows), dim3(NT), 0, s, 1, a);
    launch_k(residual_finish_kernel, dim3(a.rows), dim3(32), 0, s, 1, a, nc);
}

void launch_accept_sample(const AcceptSample &a, cudaStream_t s) {
    launch_k(accept_sample_kernel, dim3((a.nseq + 127) / 128), dim3(128), 0, s, 1, a);
}

}  // namespace dfl
