// moe_experts.cu -- MoE experts of bf16 models, touched experts only.
//
// Routing (softmax over the experts, top-k, weights renormalised over the k)
// leaves R*k (row, choice) pairs.  moe_bucket_kernel groups the pairs by expert
// and lists the experts at least one pair routes to.  At decode sizes an expert
// sees one to a few rows, so the two expert products are weight-streaming
// GEMVs bound by HBM bandwidth: each touched expert's weights are read exactly
// once per layer, untouched experts not at all.
//
// Two kernel pairs share the bucketing.  For sparse routing (decode: at most
// two pairs per expert on average), moe_stream_kernel: one CTA per SM walks a
// contiguous range of work items (touched expert, chunk of weight rows) in
// expert-major order.  A chunk's
// weight rows are contiguous in memory and arrive in shared memory through
// cp.async.bulk copies on a ring of mbarrier stages, issued ahead by one
// thread with an L2 evict-first policy, so several stages per SM are in flight
// while the warps compute.  The expert's activation rows are staged in fp32
// (both bf16 planes summed) once per expert, XR at a time; an expert with more
// rows is processed in passes that restage them.  Each warp takes one weight
// row (gate/up) or two (down) and reduces its dot products across lanes.
//   gate/up item: 4 columns f of one expert = 4 gate rows + 4 up rows,
//                 h[pair][f] = SiLU(W_gate[f] . x[row]) * (W_up[f] . x[row])
//   down item:    16 output rows o,  part[pair][o] = W_down[o] . h[pair]
// Every wait is bounded (error bit 4 after two seconds); a CTA that gives up
// waits, again bounded, for its copies in flight before it exits.
// For dense routing (prefill chunks, large batches) the row-parallel kernels
// moe_gateup_kernel / moe_down_kernel keep weight rows in registers and reuse
// them across all of the expert's rows.
#include <algorithm>

#include "kernels.h"
#include "launch.h"
#include "tc_device.cuh"

namespace dfl {

namespace {

constexpr int XR = 4;           // expert rows staged per pass
constexpr int MAX_CPL = 12;     // 16-byte chunks per lane and weight row (rows of up to 3072 bf16)
constexpr int MAX_STAGES = 8;
constexpr int NTHREADS = 256;   // 8 warps
constexpr int CTAS_PER_SM = 2;  // two independent item chains per SM
constexpr size_t SMEM_BUDGET = 110 * 1024;

struct MoeStream {
    const bf16 *x;      // activation rows: m[row] (gate/up; row = pair / k) or h[pair] (down)
    int ldx;
    size_t xlo;         // lo-plane offset of x in elements (0: one plane)
    int div;            // pair -> x row divisor (k for gate/up, 1 for down)
    const int *off;     // [E + 1] pair ranges of list per expert
    const int *list;    // [R * k] pairs grouped by expert
    const int *touched; // [E + 1] touched experts; touched[E] = their count
    const bf16 *w;      // we_gate_up [E][2 Fe][H] or we_down [E][H][Fe]
    int H, Fe, E;
    bf16 *h;            // gate/up output h[pair][Fe]
    size_t hlo;
    float *part;        // down output part[pair][H]
    int stages;
    int *err;
};

// pairs rk = r*k + t grouped by expert: off[e] .. off[e+1]-1 index list[];
// touched[0 .. nt) = experts with at least one pair (ascending), touched[E] = nt
__global__ void moe_bucket_kernel(const int *__restrict__ sel, int n_pairs, int E, int *off, int *list,
                                  int *touched) {
    pdl_trigger();
    pdl_wait();
    __shared__ int cnt[257], cur[256];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n_pairs; i += blockDim.x) atomicAdd(&cnt[sel[i]], 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0, nt = 0;
        for (int e = 0; e < E; ++e) {
            const int c = cnt[e];
            if (c) touched[nt++] = e;
            cnt[e] = acc;
            cur[e] = acc;
            acc += c;
        }
        for (int e = nt; e < E; ++e) touched[e] = -1;
        touched[E] = nt;
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

// contiguous global -> shared copy completing on an mbarrier (16-byte aligned, bytes % 16 == 0)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(tc::smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)), "l"(pol)
        : "memory");
}

// x rows of pairs list[p .. p+nc) into xs[j][0..n) in fp32 (both planes summed) and
// the pair ids into pair[0..nc): all 16-byte loads of a column chunk issued before use
__device__ __forceinline__ void stage_rows(const MoeStream &a, int p, int nc, int n, float *xs, int *pair) {
    int row[XR];
#pragma unroll
    for (int j = 0; j < XR; ++j) {
        const int pr = j < nc ? a.list[p + j] : 0;
        row[j] = pr / a.div;
        if (j < nc && threadIdx.x == 0) pair[j] = pr;
    }
    for (int c = threadIdx.x; c < n / 8; c += NTHREADS) {
        uint4 hi[XR], lw[XR];
#pragma unroll
        for (int j = 0; j < XR; ++j) {
            if (j >= nc) break;
            const size_t at = (size_t)row[j] * a.ldx + (size_t)c * 8;
            hi[j] = *reinterpret_cast<const uint4 *>(a.x + at);
            if (a.xlo) lw[j] = *reinterpret_cast<const uint4 *>(a.x + a.xlo + at);
        }
#pragma unroll
        for (int j = 0; j < XR; ++j) {
            if (j >= nc) break;
            float v[8], u[8];
            bf16x8_to_f(hi[j], v);
            if (a.xlo) {
                bf16x8_to_f(lw[j], u);
#pragma unroll
                for (int t = 0; t < 8; ++t) v[t] += u[t];
            }
            float4 *d = reinterpret_cast<float4 *>(xs + (size_t)j * n + c * 8);
            d[0] = make_float4(v[0], v[1], v[2], v[3]);
            d[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
    }
}

// ------------------------------------------------------------------------
// Row-parallel experts, for dense routing (prefill chunks, large batches): one
// CTA per (expert, 8 weight rows), grid (E, rows / 8); each warp holds its
// weight rows in registers and applies them to all of the expert's rows,
// MOE_PC at a time.  CTAs of untouched experts exit at once.
// ------------------------------------------------------------------------
constexpr int MOE_PC = 4;  // expert rows staged per pass
constexpr int MOE_CPL = MAX_CPL;  // 16-byte weight chunks per lane and row (rows of up to 3072 bf16)

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

// ------------------------------------------------------------------------
// Weight-streaming experts, for sparse routing (decode): see the file header.
// ------------------------------------------------------------------------
template <bool GU>
__global__ void __launch_bounds__(NTHREADS, CTAS_PER_SM) moe_stream_kernel(const MoeStream a) {
    pdl_trigger();
    extern __shared__ __align__(128) unsigned char sm[];
    constexpr int ROWS = GU ? 8 : 16;  // weight rows per item
    constexpr int RPW = ROWS / 8;      // weight rows per warp
    const int n = GU ? a.H : a.Fe;     // dot length = weight row length
    const int nch = GU ? a.Fe / 4 : a.H / 16;
    const uint32_t sb = (uint32_t)ROWS * n * 2;
    const int S = a.stages;
    unsigned char *wst = sm;
    float *xs = reinterpret_cast<float *>(sm + (size_t)S * sb);
    uint64_t *full = reinterpret_cast<uint64_t *>(xs + (size_t)XR * n);
    float *red = reinterpret_cast<float *>(full + MAX_STAGES);  // [2][8][XR]
    int *pair_s = reinterpret_cast<int *>(red + 2 * 8 * XR);     // [2][XR]
    int *off_s = pair_s + 2 * XR;                               // [E + 1]
    int *tch_s = off_s + a.E + 1;                               // [E + 1]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    pdl_wait();
    for (int i = tid; i <= a.E; i += NTHREADS) {
        off_s[i] = a.off[i];
        tch_s[i] = a.touched[i];
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) tc::mbar_init(&full[s], 1);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    const long long total = (long long)tch_s[a.E] * nch;
    const int j0 = (int)(total * blockIdx.x / gridDim.x), j1 = (int)(total * (blockIdx.x + 1) / gridDim.x);
    const int cnt = j1 - j0;
    if (cnt <= 0) return;

    // item j0 + q into stage q % S (thread 0 only)
    const uint64_t pol = tc::l2_evict_first_policy();
    auto issue = [&](int q) {
        const int j = j0 + q, t = j / nch, c = j - t * nch, e = tch_s[t];
        uint64_t *bar = &full[q % S];
        unsigned char *dst = wst + (size_t)(q % S) * sb;
        tc::mbar_expect_tx(bar, sb);
        if (GU) {
            const uint32_t half = sb / 2;
            bulk_g2s(dst, a.w + ((size_t)e * 2 * a.Fe + (size_t)c * 4) * n, half, bar, pol);
            bulk_g2s(dst + half, a.w + ((size_t)e * 2 * a.Fe + a.Fe + (size_t)c * 4) * n, half, bar, pol);
        } else {
            bulk_g2s(dst, a.w + ((size_t)e * a.H + (size_t)c * 16) * n, sb, bar, pol);
        }
    };
    int issued = 0;
    if (tid == 0)
        for (; issued < min(S, cnt); ++issued) issue(issued);

    const int cpl = n >> 8;
    int cur_e = -1, xv = 0, rb = 0, failed_q = -1;
    for (int q = 0; q < cnt && failed_q < 0; ++q) {
        const int j = j0 + q, t = j / nch, c = j - t * nch, e = tch_s[t];
        const int p0 = off_s[e], np = off_s[e + 1] - p0;
        const bool got = tc::mbar_wait(&full[q % S], (q / S) & 1, a.err);
        const uint4 *ws = reinterpret_cast<const uint4 *>(wst + (size_t)(q % S) * sb);
        for (int c0 = 0; c0 < np; c0 += XR) {
            const int nc = min(XR, np - c0);
            if (e != cur_e || np > XR) {
                xv ^= 1;
                stage_rows(a, p0 + c0, nc, n, xs, pair_s + xv * XR);
            }
            if (__syncthreads_or(!got)) {
                failed_q = q;
                break;
            }
            float acc[RPW][XR];
#pragma unroll
            for (int u = 0; u < RPW; ++u)
#pragma unroll
                for (int jj = 0; jj < XR; ++jj) acc[u][jj] = 0.f;
#pragma unroll
            for (int qq = 0; qq < MAX_CPL; ++qq) {
                if (qq >= cpl) break;
                const int ch = qq * 32 + lane;
                float wf[RPW][8];
#pragma unroll
                for (int u = 0; u < RPW; ++u) bf16x8_to_f(ws[(size_t)(warp + 8 * u) * (n >> 3) + ch], wf[u]);
#pragma unroll
                for (int jj = 0; jj < XR; ++jj) {
                    if (jj >= nc) break;
                    const float4 x0 = *reinterpret_cast<const float4 *>(xs + (size_t)jj * n + ch * 8);
                    const float4 x1 = *reinterpret_cast<const float4 *>(xs + (size_t)jj * n + ch * 8 + 4);
#pragma unroll
                    for (int u = 0; u < RPW; ++u)
                        acc[u][jj] += wf[u][0] * x0.x + wf[u][1] * x0.y + wf[u][2] * x0.z + wf[u][3] * x0.w +
                                      wf[u][4] * x1.x + wf[u][5] * x1.y + wf[u][6] * x1.z + wf[u][7] * x1.w;
                }
            }
            const int *pr = pair_s + xv * XR;
#pragma unroll
            for (int u = 0; u < RPW; ++u)
#pragma unroll
                for (int jj = 0; jj < XR; ++jj) {
                    if (jj >= nc) break;
                    const float v = warp_sum(acc[u][jj]);
                    if (lane == 0) {
                        if (GU)
                            red[(rb * 8 + warp) * XR + jj] = v;
                        else
                            a.part[(size_t)pr[jj] * a.H + c * 16 + warp + 8 * u] = v;
                    }
                }
            __syncthreads();
            // the item's stage is free after its last pass: refill it with item q + S
            if (tid == 0 && c0 + XR >= np && issued < cnt) issue(issued++);
            if (GU && tid < 4 * nc) {
                const int col = tid & 3, jj = tid >> 2;
                const float g = red[(rb * 8 + col) * XR + jj], up = red[(rb * 8 + 4 + col) * XR + jj];
                st_act(a.h, (size_t)pr[jj] * a.Fe + c * 4 + col, a.hlo, silu_f(g) * up);
            }
            rb ^= 1;
        }
        cur_e = e;
    }
    if (failed_q >= 0 && tid == 0) {
        // copies still in flight land before the CTA's shared memory is released
        for (int r = failed_q; r < issued; ++r) tc::mbar_wait(&full[r % S], (r / S) & 1, nullptr);
    }
}

size_t stream_smem(int n, int rows, int E, int stages) {
    return (size_t)stages * rows * n * 2 + (size_t)XR * n * 4 + MAX_STAGES * 8 + 2 * 8 * XR * 4 + 2 * XR * 4 +
           2 * (size_t)(E + 1) * 4;
}

int stream_stages(int n, int rows, int E) {
    const size_t fixed = stream_smem(n, rows, E, 0), sb = (size_t)rows * n * 2;
    return fixed < SMEM_BUDGET ? (int)std::min<size_t>(MAX_STAGES, (SMEM_BUDGET - fixed) / sb) : 0;
}

}  // namespace

// xg[pos] = m[list[pos] / k], both planes: one CTA per pair, 16-byte copies
__global__ void moe_gather_kernel(const bf16 *__restrict__ m, int ldm, size_t lo, const int *__restrict__ list, int k,
                                  int H, bf16 *__restrict__ xg) {
    pdl_trigger();
    pdl_wait();
    const int pos = blockIdx.x;
    const int row = list[pos] / k;
    const uint4 *src = reinterpret_cast<const uint4 *>(m + (size_t)row * ldm);
    uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)pos * H);
    for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
        dst[c] = src[c];
        if (lo) reinterpret_cast<uint4 *>(xg + lo + (size_t)pos * H)[c] = reinterpret_cast<const uint4 *>(m + lo + (size_t)row * ldm)[c];
    }
}

void launch_moe_gather(const bf16 *m, int ldm, size_t lo, const int *list, int k, int n_pairs, int H, bf16 *xg,
                       cudaStream_t s) {
    if (n_pairs <= 0) return;
    launch_k(moe_gather_kernel, dim3(n_pairs), dim3(128), 0, s, 1, m, ldm, lo, list, k, H, xg);
}

bool moe_bucketed_supported(int H, int Fe, int E) {
    return H % 256 == 0 && Fe % 256 == 0 && H <= 256 * MAX_CPL && Fe <= 256 * MAX_CPL && E <= 256;
}

void launch_moe_bucket(const int *sel, int n_pairs, int E, int *off, int *list, cudaStream_t s) {
    launch_k(moe_bucket_kernel, dim3(1), dim3(1024), 0, s, 1, sel, n_pairs, E, off, list, off + E + 1);
}

void launch_moe_experts_bucketed(const bf16 *m, int ldm, size_t lo, int R, int k, const int *sel, int E,
                                 const bf16 *w_gate_up, const bf16 *w_down, int H, int Fe, int *off, int *list,
                                 bf16 *h, size_t hlo, float *part, int num_sms, int *err, cudaStream_t s) {
    if (R <= 0) return;
    ensure_smem_attr((const void *)moe_stream_kernel<true>);
    ensure_smem_attr((const void *)moe_stream_kernel<false>);
    int *touched = off + E + 1;
    launch_k(moe_bucket_kernel, dim3(1), dim3(1024), 0, s, 1, sel, R * k, E, off, list, touched);
    // streaming for at most two pairs per expert on average; beyond that the
    // row-parallel kernels reuse each weight row held in registers across the rows
    const bool sparse = (long long)R * k <= 2LL * E;
    if (!sparse || stream_stages(H, 8, E) < 2 || stream_stages(Fe, 16, E) < 2) {
        launch_k(moe_gateup_kernel<bf16>, dim3(E, (Fe + 7) / 8), dim3(256), sizeof(float) * MOE_PC * H, s, 1, m, ldm,
                 lo, k, (const int *)off, (const int *)list, w_gate_up, H, Fe, h, hlo);
        launch_k(moe_down_kernel<bf16>, dim3(E, (H + 7) / 8), dim3(256), sizeof(float) * MOE_PC * Fe, s, 1,
                 (const bf16 *)h, hlo, (const int *)off, (const int *)list, w_down, H, Fe, part);
        return;
    }
    MoeStream a = {};
    a.x = m;
    a.ldx = ldm;
    a.xlo = lo;
    a.div = k;
    a.off = off;
    a.list = list;
    a.touched = touched;
    a.w = w_gate_up;
    a.H = H;
    a.Fe = Fe;
    a.E = E;
    a.h = h;
    a.hlo = hlo;
    a.part = part;
    a.err = err;
    a.stages = stream_stages(H, 8, E);
    launch_k(moe_stream_kernel<true>, dim3(CTAS_PER_SM * num_sms), dim3(NTHREADS), stream_smem(H, 8, E, a.stages), s, 1, a);
    MoeStream d = a;
    d.x = h;
    d.ldx = Fe;
    d.xlo = hlo;
    d.div = 1;
    d.w = w_down;
    d.stages = stream_stages(Fe, 16, E);
    launch_k(moe_stream_kernel<false>, dim3(CTAS_PER_SM * num_sms), dim3(NTHREADS), stream_smem(Fe, 16, E, d.stages), s, 1, d);
}

}  // namespace dfl
