// attn_mma.cu -- block attention for bf16 models on tensor cores (mma.sync
// m16n8k16, fp32 accumulate, online softmax), with split-KV across CTAs.
//
// One CTA serves one query tile (up to 16 consecutive rows of one sequence:
// a draft/verify block, or 16 prompt rows) for one KV head and one share of
// its keys; its warps are the q heads that share that KV head (GQA), in one or
// two key groups, so each K/V tile is read from HBM once for the whole group.
// Row r sees keys [0, meta[r].nk): the target's verify rows are causal
// (nk = pos + 1), the drafter's block rows are block-bidirectional (nk = p + B:
// every committed context key and every key of the block) -- "O que o DFlash
// faz de diferente" on the iaemfoco DFlash page (the drafter fills the whole
// block in one parallel pass).
//
// The visible keys are cut into n_splits shares (CTAs of one cluster); every
// warp keeps an unnormalised partial (o, running max, running sum), pushes it
// into the shared memory of the CTA that finishes its (head, row) pair, and
// after one cluster barrier each CTA combines its pairs over all partials in a
// fixed order (deterministic).  At 16 query rows the products are small; the
// legacy tensor-core path (mma.sync) covers them, the projections use tcgen05.
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

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ const float *peer_ptr(const float *p, uint32_t rank) {
    uint64_t out;
    asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const float *>(out);
}

// store 2 floats (8-byte aligned) to the same shared-memory location in CTA `rank`
__device__ __forceinline__ void st_cluster_v2(float *local, uint32_t rank, float a, float b) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(ra), "f"(a), "f"(b) : "memory");
}

// bounded wait until *p >= target (acquire); error bit 16 after 2 s
__device__ __forceinline__ void wait_ctr(const int *p, int target, int *err) {
    auto ld = [&] {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v;
    };
    if (ld() >= target) return;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (ld() >= target) return;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > 2000000000ull) {
            if (err) atomicOr(err, 16);
            return;
        }
        __nanosleep(32);
    }
}

__device__ __forceinline__ void group_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One CTA serves one (query tile, kv head, KV split); the n_splits CTAs of a
// (tile, kv head) form a cluster along z.  A CTA's warps are G key groups of
// `grp` warps, one warp per q head of the kv head (GQA): key group g takes key
// tiles g, g+G, ... of the split's share, each tile loaded once into the
// group's own buffer and read by all its heads.  Every warp ends with an
// unnormalised partial (o, running max, running sum) for its head and rows;
// it pushes that partial into the shared memory of the CTA that finishes the
// (head, row) pair ("owner"), so after one cluster barrier each CTA combines
// its pairs from local memory over all n_splits * G partials in a fixed order
// (identical results run to run).
//
// SPLIT: q, K, V (and the output) are two-plane activations (hi at p, lo at
// p + lo).  Each product then takes three bf16 MMAs, hi*hi + lo*hi + hi*lo
// (the lo*lo term is below the fp32 accumulator's resolution), and the
// probabilities P are split the same way in registers before P V.
template <int HD, bool SPLIT>
__global__ void __launch_bounds__(256) attn_mma_kernel(const bf16 *__restrict__ q, int ldq, const bf16 *__restrict__ kc,
                                                       const bf16 *__restrict__ vc, const RowMeta *__restrict__ meta,
                                                       int R, int rows_per_tile, int nq, int nkv, int max_len,
                                                       int n_splits, int G, float scale_log2, bf16 *__restrict__ out,
                                                       int ldo, size_t lo, const int *dep_ctr, int dep_target,
                                                       int *done_ctr, int *err) {
    constexpr int LDS = HD + 8;                 // padded smem row (bf16 elements)
    constexpr int NPL = SPLIT ? 4 : 2;          // planes per tile buffer: K, V (+ K lo, V lo)
    constexpr int PLANE = KB * LDS;             // elements of one plane of a tile buffer
    extern __shared__ __align__(16) uint8_t smem_raw[];

    // every CTA of the cluster has started before any CTA stores into another's
    // shared memory: arrive now, wait before the first push
    cluster_arrive_relaxed();
    pdl_trigger();
    if (dep_ctr) {  // completion counter of the projection that wrote q and K/V
        if (threadIdx.x == 0) wait_ctr(dep_ctr, dep_target, err);
        __syncthreads();
    } else {
        pdl_wait();
    }
    const int tile = blockIdx.x, kvh = blockIdx.y, split = blockIdx.z;
    const int grp = nq / nkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hw = warp % grp, g = warp / grp;  // head within the kv group, key group
    const int gthr = 32 * grp;                  // threads of one key group
    const int gt = threadIdx.x - g * gthr;
    const int r0 = tile * rows_per_tile;
    const int nrows = min(rows_per_tile, R - r0);
    const int seq = meta[r0].seq;
    const int h = kvh * grp + hw;
    const int pairs = grp * 16, ppc = (pairs + n_splits - 1) / n_splits;  // (head, row) pairs per owner
    const int nsrc = n_splits * G;                                       // partials per pair
    bf16 *tb = reinterpret_cast<bf16 *>(smem_raw) + (size_t)g * NPL * PLANE;
    float *recv_o = reinterpret_cast<float *>(smem_raw + (size_t)G * NPL * PLANE * sizeof(bf16));  // [nsrc][ppc][HD]
    float *recv_ml = recv_o + (size_t)nsrc * ppc * HD;                                               // [nsrc][ppc][2]

    // visible keys of the two rows this thread's accumulators cover
    const int ra = lane >> 2, rb = ra + 8;
    const int nk_a = ra < nrows ? meta[r0 + ra].nk : 0;
    const int nk_b = rb < nrows ? meta[r0 + rb].nk : 0;
    // longest visible key range of the tile's rows (nrows <= 16), the same in every lane
    int nk_max = lane < nrows ? meta[r0 + lane].nk : 0;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) nk_max = max(nk_max, __shfl_xor_sync(0xffffffffu, nk_max, o2));
    // this split's key tiles [t0, t1); key group g takes t0 + g, t0 + g + G, ...
    const int ntk = (nk_max + KB - 1) / KB;
    const int per = (ntk + n_splits - 1) / n_splits;
    const int t0 = min(ntk, split * per), t1 = min(ntk, t0 + per);

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

    const bf16 *Kt = tb, *Vt = tb + PLANE, *Klt = tb + 2 * PLANE, *Vlt = tb + 3 * PLANE;
#pragma unroll 1
    for (int tt = t0 + g; tt < t1; tt += G) {
        const int j0 = tt * KB;
        {
            constexpr int CPR = HD / 8;  // 16-byte chunks per row
            bf16 *Kw = tb, *Vw = tb + PLANE;
#pragma unroll 1
            for (int e = gt; e < KB * CPR; e += gthr) {
                const int r = e / CPR, c = (e % CPR) * 8;
                const int key = j0 + r;
                const bool valid = key < nk_max;
                const size_t off = (size_t)(valid ? key : 0) * HD + c;
                cp_async16(Kw + r * LDS + c, Kg + off, valid);
                cp_async16(Vw + r * LDS + c, Vg + off, valid);
                if constexpr (SPLIT) {
                    cp_async16(Kw + 2 * PLANE + r * LDS + c, Kg + lo + off, valid);
                    cp_async16(Vw + 2 * PLANE + r * LDS + c, Vg + lo + off, valid);
                }
            }
            cp_commit();
            cp_wait<0>();
        }
        group_bar(1 + g, gthr);
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
        group_bar(1 + g, gthr);  // the buffer is reloaded by the next tile
    }
    // row sums across the quad
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

    // ---- push this warp's partial to the owners of its (head, row) pairs ----
    cluster_wait();
    const int src = split * G + g;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int row = half ? rb : ra;
        if (row >= nrows) continue;
        const int pair = hw * 16 + row, owner = pair / ppc, pl = pair - owner * ppc;
        float *dst = recv_o + ((size_t)src * ppc + pl) * HD + (lane & 3) * 2;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j)
            st_cluster_v2(dst + j * 8, (uint32_t)owner, o[j][2 * half], o[j][2 * half + 1]);
        if ((lane & 3) == 0)
            st_cluster_v2(recv_ml + ((size_t)src * ppc + pl) * 2, (uint32_t)owner, half ? m_b : m_a, half ? l_b : l_a);
    }
    __syncwarp();
    cluster_sync_all();  // (a 1-CTA cluster when n_splits == 1)

    // ---- combine the owned pairs over all partials, in source order ----
    const int p0 = split * ppc, p1 = min(pairs, p0 + ppc);
    constexpr int D4 = HD / 4;
#pragma unroll 1
    for (int e = threadIdx.x; e < (p1 - p0) * D4; e += blockDim.x) {
        const int pl = e / D4, d0 = (e % D4) * 4;
        const int pair = p0 + pl, hh = pair / 16, row = pair % 16;
        if (row >= nrows) continue;
        float mstar = -INFINITY;
#pragma unroll 1
        for (int s2 = 0; s2 < nsrc; ++s2) mstar = fmaxf(mstar, recv_ml[((size_t)s2 * ppc + pl) * 2]);
        const float mu = mstar == -INFINITY ? 0.f : mstar;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lsum = 0.f;
#pragma unroll 1
        for (int s2 = 0; s2 < nsrc; ++s2) {
            const float2 ml = *reinterpret_cast<const float2 *>(recv_ml + ((size_t)s2 * ppc + pl) * 2);
            const float w = exp2f(ml.x - mu);
            const float4 v = *reinterpret_cast<const float4 *>(recv_o + ((size_t)s2 * ppc + pl) * HD + d0);
            lsum += ml.y * w;
            acc.x += v.x * w;
            acc.y += v.y * w;
            acc.z += v.z * w;
            acc.w += v.w * w;
        }
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        bf16 *dst = out + (size_t)(r0 + row) * ldo + (kvh * grp + hh) * HD + d0;
        store_pair(dst, lo, acc.x * inv, acc.y * inv);
        store_pair(dst + 2, lo, acc.z * inv, acc.w * inv);
    }
    if (done_ctr) {  // every writer fences (generic and async proxy), then one signal per CTA
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(done_ctr, 1);
        }
    }
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

// key groups per CTA: two when the kv group has at most 4 q heads (8 warps)
static int attn_groups(int grp) { return grp <= 4 ? 2 : 1; }

static size_t attn_smem(int hd, bool split, int grp, int n_splits) {
    const int G = attn_groups(grp);
    const size_t tiles = (size_t)G * (split ? 4 : 2) * at::KB * (hd + 8) * sizeof(bf16);
    const int pairs = grp * 16, ppc = (pairs + n_splits - 1) / n_splits;
    const size_t recv = (size_t)n_splits * G * ppc * (hd + 2) * sizeof(float);
    return tiles + recv;
}

template <int HD, bool SPLIT>
static void launch_hd(const bf16 *q, int ldq, const bf16 *kc, const bf16 *vc, const RowMeta *meta, int R,
                      int rows_per_tile, int nq, int nkv, int max_len, bf16 *out, int ldo, size_t lo, int n_tiles,
                      int n_splits, const AttnSync &sy, cudaStream_t s) {
    const int grp = nq / nkv;
    const int G = attn_groups(grp);
    const size_t smem = attn_smem(HD, SPLIT, grp, n_splits);
    ensure_smem_attr((const void *)at::attn_mma_kernel<HD, SPLIT>);
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
    launch_k(at::attn_mma_kernel<HD, SPLIT>, dim3(n_tiles, nkv, n_splits), dim3(32 * grp * G), smem, s, n_splits, q, ldq,
             kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, n_splits, G, scale_log2, out, ldo, lo, sy.dep_ctr,
             sy.dep_target, sy.done_ctr, sy.err);
}

template <>
int launch_attention_mma<bf16>(const bf16 *q, int ldq, const bf16 *kc, const bf16 *vc, const RowMeta *meta, int R,
                               int rows_per_tile, int nq, int nkv, int hd, int max_len, bf16 *out, int ldo, size_t lo,
                               const AttnScratch &ws, cudaStream_t s, const AttnSync &sy) {
    if (R <= 0) return 0;
    const int g_num_sms = ws.num_sms;
    const int n_tiles = (R + rows_per_tile - 1) / rows_per_tile;
    const int ctas = n_tiles * nkv;
    // splits of one (tile, kv head) form a cluster of at most 8 CTAs; no more
    // splits than 64-key tiles the longest possible context has
    const int n_splits = std::max(1, std::min({8, (2 * g_num_sms + ctas - 1) / ctas, (max_len + 63) / 64}));
    if (hd == 128) {
        if (lo) launch_hd<128, true>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, lo, n_tiles, n_splits, sy, s);
        else launch_hd<128, false>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, 0, n_tiles, n_splits, sy, s);
    } else {
        if (lo) launch_hd<64, true>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, lo, n_tiles, n_splits, sy, s);
        else launch_hd<64, false>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len, out, ldo, 0, n_tiles, n_splits, sy, s);
    }
    return n_tiles * nkv * n_splits;
}

template <>
int launch_attention_mma<float>(const float *, int, const float *, const float *, const RowMeta *, int, int, int, int,
                                int, int, float *, int, size_t, const AttnScratch &, cudaStream_t, const AttnSync &) {
    return 0;
}

}  // namespace dfl
