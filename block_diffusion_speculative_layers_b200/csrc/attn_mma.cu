// attn_mma.cu -- block attention for bf16 models on tensor cores (mma.sync
// m16n8k16, fp32 accumulate, online softmax), with split-KV across CTAs.
//
// One CTA serves one query tile (up to 16 consecutive rows of one sequence:
// a draft/verify block, or 16 prompt rows) for one KV head; its warps are the
// q heads that share that KV head (GQA), so each K/V tile is read from HBM once
// for the whole group.  Row r sees keys [0, meta[r].nk): the target's verify
// rows are causal (nk = pos + 1), the drafter's block rows are
// block-bidirectional (nk = p + B: every committed context key and every key
// of the block) -- "O que o DFlash faz de diferente" on the iaemfoco DFlash
// page (the drafter fills the whole block in one parallel pass).
//
// The KV range [0, max_len) is cut into n_splits chunks; each CTA writes an
// unnormalised partial (o, running max, running sum) and the last CTA of the
// (tile, kv head) combines the partials in split order (deterministic).
// Attention reads K/V once per group and is bound by HBM traffic, which the
// legacy tensor-core path covers; the projections use tcgen05 (gemm_tc.cu).
#include <math.h>

#include "attn_mma.h"
#include "launch.h"

namespace dfl {
namespace at {

constexpr int KB = 64;  // keys per smem tile

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// (a, b) as a bf16 pair of high parts and a bf16 pair of the rounding remainders
__device__ __forceinline__ void split_pack(float a, float b, uint32_t &hi, uint32_t &rem) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    const __nv_bfloat162 r = __floats2bfloat162_rn(a - __low2float(h), b - __high2float(h));
    rem = *reinterpret_cast<const uint32_t *>(&r);
}

// two consecutive outputs, with their low plane `lo` elements further on when lo != 0
__device__ __forceinline__ void store_pair(bf16 *dst, size_t lo, float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    *reinterpret_cast<__nv_bfloat162 *>(dst) = h;
    if (lo) *reinterpret_cast<__nv_bfloat162 *>(dst + lo) = __floats2bfloat162_rn(a - __low2float(h), b - __high2float(h));
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ const float *peer_ptr(const float *p, uint32_t rank) {
    uint64_t out;
    asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const float *>(out);
}

// The n_splits CTAs of one (query tile, kv head) form a cluster along z.  Each
// takes an equal share of the visible keys (chunk sized on the device from the
// tile's key count), keeps an unnormalised partial (o, running max, running
// sum) in shared memory, and after a cluster barrier combines a slice of the
// (head, row) pairs over all CTAs of the cluster in rank order.
//
// SPLIT: q, K, V (and the output) are two-plane activations (hi at p, lo at
// p + lo).  Each product then takes three bf16 MMAs, hi*hi + lo*hi + hi*lo
// (the lo*lo term is below the fp32 accumulator's resolution), and the
// probabilities P are split the same way in registers before P V.
template <int HD, bool SPLIT>
__global__ void __launch_bounds__(256) attn_mma_kernel(const bf16 *__restrict__ q, int ldq, const bf16 *__restrict__ kc,
                                                       const bf16 *__restrict__ vc, const RowMeta *__restrict__ meta,
                                                       int R, int rows_per_tile, int nq, int nkv, int max_len,
                                                       int n_splits, float scale_log2, bf16 *__restrict__ out, int ldo,
                                                       size_t lo) {
    constexpr int LDS = HD + 8;  // padded smem row (bf16 elements)
    constexpr int OLD = HD + 4;  // partial-output row stride (floats)
    extern __shared__ __align__(16) uint8_t smem_raw[];
    bf16 *Ks = reinterpret_cast<bf16 *>(smem_raw);  // [2][KB][LDS]
    bf16 *Vs = Ks + 2 * KB * LDS;                    // [2][KB][LDS]
    bf16 *Kl = Vs + 2 * KB * LDS;                    // SPLIT: lo planes [2][KB][LDS] each
    bf16 *Vl = Kl + 2 * KB * LDS;
    float *Op = reinterpret_cast<float *>(smem_raw); // [grp][16][OLD], reuses K/V tiles after the loop
    __shared__ float MLs[8 * 16 * 2];                // [grp][16][(max, sum)]

    pdl_trigger();
    pdl_wait();
    const int tile = blockIdx.x, kvh = blockIdx.y, split = blockIdx.z;
    const int grp = nq / nkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthr = blockDim.x;
    const int r0 = tile * rows_per_tile;
    const int nrows = min(rows_per_tile, R - r0);
    const int seq = meta[r0].seq;
    const int h = kvh * grp + warp;

    // visible keys of the two rows this thread's accumulators cover
    const int ra = lane >> 2, rb = ra + 8;
    const int nk_a = ra < nrows ? meta[r0 + ra].nk : 0;
    const int nk_b = rb < nrows ? meta[r0 + rb].nk : 0;
    int nk_max = 0;
    for (int i = 0; i < nrows; ++i) nk_max = max(nk_max, meta[r0 + i].nk);
    // equal share of the visible keys for each split, in whole 64-key tiles
    const int chunk = ((nk_max + n_splits - 1) / n_splits + KB - 1) / KB * KB;
    const int kb = split * chunk;
    const int ke = min(kb + chunk, nk_max);

    const size_t head_off = ((size_t)seq * nkv + kvh) * (size_t)max_len * HD;
    const bf16 *Kg = kc + head_off;
    const bf16 *Vg = vc + head_off;

    // Q fragments (A operand, 16 rows x HD); ql: lo plane
    uint32_t qa[HD / 16][4], ql[SPLIT ? HD / 16 : 1][4];
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const int c0 = kk * 16 + (lane & 3) * 2;
        const bf16 *qa_row = q + (size_t)(r0 + ra) * ldq + h * HD;
        const bf16 *qb_row = q + (size_t)(r0 + rb) * ldq + h * HD;
        qa[kk][0] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0) : 0u;
        qa[kk][1] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0) : 0u;
        qa[kk][2] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0 + 8) : 0u;
        qa[kk][3] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0 + 8) : 0u;
        if constexpr (SPLIT) {
            ql[kk][0] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + lo + c0) : 0u;
            ql[kk][1] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + lo + c0) : 0u;
            ql[kk][2] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + lo + c0 + 8) : 0u;
            ql[kk][3] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + lo + c0 + 8) : 0u;
        }
    }

    float o[HD / 8][4];
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    auto load_tile = [&](int buf, int j0) {
        constexpr int CPR = HD / 8;  // 16-byte chunks per row
        for (int e = threadIdx.x; e < KB * CPR; e += nthr) {
            const int r = e / CPR, c = (e % CPR) * 8;
            const int key = j0 + r;
            const bool valid = key < ke;
            const size_t off = (size_t)(valid ? key : 0) * HD + c;
            cp_async16(Ks + ((size_t)buf * KB + r) * LDS + c, Kg + off, valid);
            cp_async16(Vs + ((size_t)buf * KB + r) * LDS + c, Vg + off, valid);
            if constexpr (SPLIT) {
                cp_async16(Kl + ((size_t)buf * KB + r) * LDS + c, Kg + lo + off, valid);
                cp_async16(Vl + ((size_t)buf * KB + r) * LDS + c, Vg + lo + off, valid);
            }
        }
        cp_commit();
    };

    const int n_blocks = ke > kb ? (ke - kb + KB - 1) / KB : 0;
    if (n_blocks > 0) load_tile(0, kb);
    for (int bi = 0; bi < n_blocks; ++bi) {
        const int buf = bi & 1;
        const int j0 = kb + bi * KB;
        if (bi + 1 < n_blocks) {
            load_tile(buf ^ 1, j0 + KB);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        const bf16 *Kt = Ks + (size_t)buf * KB * LDS;
        const bf16 *Vt = Vs + (size_t)buf * KB * LDS;
        const bf16 *Klt = Kl + (size_t)buf * KB * LDS;
        const bf16 *Vlt = Vl + (size_t)buf * KB * LDS;
        // S = Q K^T over 64 keys: 8 n-tiles of 8 keys
        float sc[KB / 8][4];
#pragma unroll
        for (int nt = 0; nt < KB / 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < KB / 16; ++np) {
                // two n-tiles (16 keys) x 16 dims: matrices (keys 0-7, d 0-7), (keys 0-7, d 8-15),
                // (keys 8-15, d 0-7), (keys 8-15, d 8-15)
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
                uint32_t b0, b1, b2, b3;
                ldm_x4(b0, b1, b2, b3, Kt + (size_t)key * LDS + dim);
                mma16816(sc[2 * np], qa[kk], b0, b1);
                mma16816(sc[2 * np + 1], qa[kk], b2, b3);
                if constexpr (SPLIT) {
                    mma16816(sc[2 * np], ql[kk], b0, b1);
                    mma16816(sc[2 * np + 1], ql[kk], b2, b3);
                    ldm_x4(b0, b1, b2, b3, Klt + (size_t)key * LDS + dim);
                    mma16816(sc[2 * np], qa[kk], b0, b1);
                    mma16816(sc[2 * np + 1], qa[kk], b2, b3);
                }
            }
        }
        // mask + online softmax (log2 domain)
        float mx_a = m_a, mx_b = m_b;
#pragma unroll
        for (int nt = 0; nt < KB / 8; ++nt) {
            const int key = j0 + nt * 8 + (lane & 3) * 2;
            sc[nt][0] = key < nk_a ? sc[nt][0] * scale_log2 : -INFINITY;
            sc[nt][1] = key + 1 < nk_a ? sc[nt][1] * scale_log2 : -INFINITY;
            sc[nt][2] = key < nk_b ? sc[nt][2] * scale_log2 : -INFINITY;
            sc[nt][3] = key + 1 < nk_b ? sc[nt][3] * scale_log2 : -INFINITY;
            mx_a = fmaxf(mx_a, fmaxf(sc[nt][0], sc[nt][1]));
            mx_b = fmaxf(mx_b, fmaxf(sc[nt][2], sc[nt][3]));
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float ua = mx_a == -INFINITY ? 0.f : mx_a;
        const float ub = mx_b == -INFINITY ? 0.f : mx_b;
        const float ca = exp2f(m_a - ua), cb = exp2f(m_b - ub);
        m_a = mx_a;
        m_b = mx_b;
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int nt = 0; nt < KB / 8; ++nt) {
            sc[nt][0] = exp2f(sc[nt][0] - ua);
            sc[nt][1] = exp2f(sc[nt][1] - ua);
            sc[nt][2] = exp2f(sc[nt][2] - ub);
            sc[nt][3] = exp2f(sc[nt][3] - ub);
            sa += sc[nt][0] + sc[nt][1];
            sb += sc[nt][2] + sc[nt][3];
        }
        l_a = l_a * ca + sa;
        l_b = l_b * cb + sb;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
            o[j][0] *= ca;
            o[j][1] *= ca;
            o[j][2] *= cb;
            o[j][3] *= cb;
        }
        // O += P V : P as A operand (4 k-steps of 16 keys), V via transposed ldmatrix
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk) {
            uint32_t pa[4], pl[4];
            if constexpr (SPLIT) {
                split_pack(sc[2 * kk][0], sc[2 * kk][1], pa[0], pl[0]);
                split_pack(sc[2 * kk][2], sc[2 * kk][3], pa[1], pl[1]);
                split_pack(sc[2 * kk + 1][0], sc[2 * kk + 1][1], pa[2], pl[2]);
                split_pack(sc[2 * kk + 1][2], sc[2 * kk + 1][3], pa[3], pl[3]);
            } else {
                pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
                pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
                pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
            }
#pragma unroll
            for (int dp = 0; dp < HD / 16; ++dp) {
                // matrices (keys 0-7, d 0-7), (keys 8-15, d 0-7), (keys 0-7, d 8-15), (keys 8-15, d 8-15)
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int dim = dp * 16 + (lane >> 4) * 8;
                uint32_t b0, b1, b2, b3;
                ldm_x4_t(b0, b1, b2, b3, Vt + (size_t)key * LDS + dim);
                mma16816(o[2 * dp], pa, b0, b1);
                mma16816(o[2 * dp + 1], pa, b2, b3);
                if constexpr (SPLIT) {
                    mma16816(o[2 * dp], pl, b0, b1);
                    mma16816(o[2 * dp + 1], pl, b2, b3);
                    ldm_x4_t(b0, b1, b2, b3, Vlt + (size_t)key * LDS + dim);
                    mma16816(o[2 * dp], pa, b0, b1);
                    mma16816(o[2 * dp + 1], pa, b2, b3);
                }
            }
        }
        __syncthreads();
    }
    // row sums across the quad
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

    if (n_splits == 1) {
        const float ia = l_a > 0.f ? 1.f / l_a : 0.f, ib = l_b > 0.f ? 1.f / l_b : 0.f;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
            const int d = j * 8 + (lane & 3) * 2;
            if (ra < nrows) store_pair(out + (size_t)(r0 + ra) * ldo + h * HD + d, lo, o[j][0] * ia, o[j][1] * ia);
            if (rb < nrows) store_pair(out + (size_t)(r0 + rb) * ldo + h * HD + d, lo, o[j][2] * ib, o[j][3] * ib);
        }
        return;
    }
    // ---- cluster combine of the splits ----
    __syncthreads();  // K/V tiles are no longer read: reuse them for the partial outputs
    {
        float *ow = Op + (size_t)warp * 16 * OLD;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
            const int d = j * 8 + (lane & 3) * 2;
            ow[ra * OLD + d] = o[j][0];
            ow[ra * OLD + d + 1] = o[j][1];
            ow[rb * OLD + d] = o[j][2];
            ow[rb * OLD + d + 1] = o[j][3];
        }
        if ((lane & 3) == 0) {
            MLs[(warp * 16 + ra) * 2] = m_a;
            MLs[(warp * 16 + ra) * 2 + 1] = l_a;
            MLs[(warp * 16 + rb) * 2] = m_b;
            MLs[(warp * 16 + rb) * 2 + 1] = l_b;
        }
    }
    __syncwarp();
    cluster_sync_all();
    {
        const int rank = (int)cluster_rank();
        const int pairs = grp * 16;                       // (head, row) pairs of the tile
        const int per = (pairs + n_splits - 1) / n_splits;
        const int p0 = rank * per, p1 = min(pairs, p0 + per);
        constexpr int DPT = 8;                             // output elements per thread
        const int tpp = HD / DPT;                          // threads per pair
        for (int e = threadIdx.x; e < (p1 - p0) * tpp; e += nthr) {
            const int pr = p0 + e / tpp, d0 = (e % tpp) * DPT;
            const int hh = pr / 16, row = pr % 16;
            if (row >= nrows) continue;
            float ms[8], ls[8];
            float mstar = -INFINITY;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                if (s2 < n_splits) {
                    const float *ml = peer_ptr(MLs, (uint32_t)s2);
                    ms[s2] = ml[(hh * 16 + row) * 2];
                    ls[s2] = ml[(hh * 16 + row) * 2 + 1];
                    mstar = fmaxf(mstar, ms[s2]);
                } else {
                    ms[s2] = -INFINITY;
                    ls[s2] = 0.f;
                }
            }
            const float mu = mstar == -INFINITY ? 0.f : mstar;
            float acc[DPT];
#pragma unroll
            for (int t = 0; t < DPT; ++t) acc[t] = 0.f;
            float lsum = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                if (s2 >= n_splits) break;
                const float w = exp2f(ms[s2] - mu);
                lsum += ls[s2] * w;
                const float *src = peer_ptr(Op, (uint32_t)s2) + ((size_t)hh * 16 + row) * OLD + d0;
                const float4 a = *reinterpret_cast<const float4 *>(src);
                const float4 b = *reinterpret_cast<const float4 *>(src + 4);
                acc[0] += a.x * w; acc[1] += a.y * w; acc[2] += a.z * w; acc[3] += a.w * w;
                acc[4] += b.x * w; acc[5] += b.y * w; acc[6] += b.z * w; acc[7] += b.w * w;
            }
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
            const int hq = kvh * grp + hh;
            bf16 *dst = out + (size_t)(r0 + row) * ldo + hq * HD + d0;
#pragma unroll
            for (int t = 0; t < DPT; t += 2) store_pair(dst + t, lo, acc[t] * inv, acc[t + 1] * inv);
        }
    }
    cluster_sync_all();
}

}  // namespace at

AttnWorkspace attn_workspace_plan(int max_rows, int nq, int nkv, int max_len, int num_sms) {
    (void)max_len;
    AttnWorkspace w;
    // query tiles of a launch (at most one per row) plus the splits that fill the GPU
    const size_t tiles = (size_t)max_rows;
    const size_t split_budget = (size_t)(2 * num_sms + nkv - 1) / nkv + 1;
    w.max_parts = (tiles + split_budget) * (size_t)nq * 16;
    return w;
}

template <>
bool attn_mma_supported<bf16>(int hd) {
    return hd == 64 || hd == 128;
}
template <>
bool attn_mma_supported<float>(int) {
    return false;
}

static int g_num_sms = 0;

template <int HD, bool SPLIT>
static void launch_hd(const bf16 *q, int ldq, const bf16 *kc, const bf16 *vc, const RowMeta *meta, int R,
                      int rows_per_tile, int nq, int nkv, int max_len, bf16 *out, int ldo, size_t lo, int n_tiles,
                      int n_splits, cudaStream_t s) {
    const int grp = nq / nkv;
    size_t smem = (SPLIT ? 4 : 2) * 2 * at::KB * (HD + 8) * sizeof(bf16);
    smem = std::max(smem, (size_t)grp * 16 * (HD + 4) * sizeof(float));
    static bool set = false;
    if (!set) {
        cudaFuncSetAttribute(at::attn_mma_kernel<HD, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        set = true;
    }
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
    launch_k(at::attn_mma_kernel<HD, SPLIT>, dim3(n_tiles, nkv, n_splits), dim3(32 * grp), smem, s, n_splits, q, ldq, kc,
             vc, meta, R, rows_per_tile, nq, nkv, max_len, n_splits, scale_log2, out, ldo, lo);
}

template <>
void launch_attention_mma<bf16>(const bf16 *q, int ldq, const bf16 *kc, const bf16 *vc, const RowMeta *meta, int R,
                                int rows_per_tile, int nq, int nkv, int hd, int max_len, bf16 *out, int ldo, size_t lo,
                                const AttnScratch &ws, cudaStream_t s) {
    (void)ws;
    if (R <= 0) return;
    if (!g_num_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int n_tiles = (R + rows_per_tile - 1) / rows_per_tile;
    const int ctas = n_tiles * nkv;
    // splits of one (tile, kv head) form a cluster of at most 8 CTAs; no more
    // splits than 64-key tiles the longest possible context has
    const int n_splits = std::max(1, std::min({8, (2 * g_num_sms + ctas - 1) / ctas, (max_len + 63) / 64}));
    if (hd == 128) {
        if (lo) launch_hd<128, true>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, lo, n_tiles, n_splits, s);
        else launch_hd<128, false>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, 0, n_tiles, n_splits, s);
    } else {
        if (lo) launch_hd<64, true>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, lo, n_tiles, n_splits, s);
        else launch_hd<64, false>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, 0, n_tiles, n_splits, s);
    }
}

template <>
void launch_attention_mma<float>(const float *, int, const float *, const float *, const RowMeta *, int, int, int, int,
                                 int, int, float *, int, size_t, const AttnScratch &, cudaStream_t) {}

}  // namespace dfl
