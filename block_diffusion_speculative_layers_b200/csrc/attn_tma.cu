// attn_tma.cu -- block attention for bf16 models, tuned for the latency of a
// decode step (one block of up to 16 query rows per sequence).
//
// Row r of a query tile sees keys [0, meta[r].nk): the target's verify rows
// are causal (nk = pos + 1); the drafter's block rows are block-bidirectional
// (nk = p + B: every committed context key and every key of the block) --
// "O que o DFlash faz de diferente" on the iaemfoco DFlash page (the drafter
// fills the whole block in one parallel pass; the target checks it in one).
//
// Work split.  A CTA serves one query tile, HPC q heads of one kv head (GQA)
// and one share of the keys ("split"); the n_splits CTAs of a (tile, head
// group) form a thread-block cluster along z.  With HPC = 1 a decode step of
// one sequence has 32 q heads x 8 splits = 256 CTAs, so the K/V of a short
// context streams through every SM at once instead of through 64.
//
// Data movement.  The K and V caches are viewed as 5-D tensors (head_dim,
// position, sequence x kv head, layer, plane); one producer warp loads each
// 32-key tile with four TMA boxes {64 dims, 32 keys, 1, 1, planes} -- both
// bf16 planes of two-plane activations in one box -- 128-byte swizzled, into
// a ring of stages guarded by mbarriers.  Four consumer warps (HPC heads x
// G = 4 / HPC key groups) compute S = Q K^T and O += P V with mma.sync
// m16n8k16 (16 query rows per head: far too few for the tcgen05 tile shapes
// to pay), three products per pair for two-plane operands (hi*hi + lo*hi +
// hi*lo), online softmax in the log2 domain.
//
// Combine.  Key groups of one CTA are merged through shared memory, then each
// CTA pushes its (o, max, sum) partial of every (head, row) pair into the
// shared memory of the cluster CTA that finishes that pair; after one cluster
// barrier the owners merge the n_splits partials in split order (identical
// results run to run) and store the output rows.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA sets
// bit 32 of the device error word and carries on without the tile.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <cstdlib>

#include "attn_tma.h"
#include "launch.h"

namespace dfl {
namespace atm {

constexpr int NCW = 4;                   // consumer warps
constexpr int NTH = 32 * (NCW + 1);      // + one producer warp
constexpr unsigned long long WAIT_NS = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait: false (and error bit 32) after WAIT_NS
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, int *err) {
    if (mbar_try(b, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try(b, parity)) return true;
        if (gtimer() - t0 > WAIT_NS) {
            if (err) atomicOr(err, 32);  // bit 5: an attention wait gave up
            return false;
        }
    }
}

// one box {64, KT, 1, 1, planes} of a 5-D (or {64, KT, 1, 1} of a 4-D) K/V map
// (KT, the keys per tile, is the map's box height)
__device__ __forceinline__ void tma_box(void *dst, const CUtensorMap *map, int d0, int key, int sh, int layer,
                                        bool five, uint64_t *bar) {
    if (five)
        asm volatile(
            "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, "
            "%7}], [%2];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(d0), "r"(key), "r"(sh), "r"(layer), "r"(0)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
            "%6}], [%2];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(d0), "r"(key), "r"(sh), "r"(layer)
            : "memory");
}

// L2 prefetch of the same box (no shared memory written, no barrier)
__device__ __forceinline__ void tma_box_prefetch(const CUtensorMap *map, int d0, int key, int sh, int layer, bool five) {
    if (five)
        asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(
                         reinterpret_cast<uint64_t>(map)),
                     "r"(d0), "r"(key), "r"(sh), "r"(layer), "r"(0)
                     : "memory");
    else
        asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                         reinterpret_cast<uint64_t>(map)),
                     "r"(d0), "r"(key), "r"(sh), "r"(layer)
                     : "memory");
}

// this CTA's key tiles [t0, t1) of a query tile whose longest row sees nk_max keys
__device__ __forceinline__ void split_range(int nk_max, int KT, int S, int split, int &t0, int &t1) {
    const int ntk = (nk_max + KT - 1) / KT;
    const int per = (ntk + S - 1) / S;
    t0 = min(ntk, split * per);
    t1 = min(ntk, t0 + per);
}

__device__ __forceinline__ void ldm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
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
// store 2 floats (8-byte aligned) to the same shared-memory location in CTA `rank`
__device__ __forceinline__ void st_cluster_v2(float *local, uint32_t rank, float a, float b) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(ra), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(float *local, uint32_t rank, float4 v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

// byte offset of (key, dim) in one swizzled box region [keys][64 dims] (128-byte
// rows; 16-byte chunk c of row k stored at chunk c ^ (k & 7))
__device__ __forceinline__ uint32_t swz(int key, int dim64) {
    return (uint32_t)(key * 128 + ((((dim64 >> 3) ^ key) & 7) << 4) + (dim64 & 7) * 2);
}

// Stage layout: [K box 0][K box 1][V box 0][V box 1], each box [planes][KT][128 B]
// (dims 64*box .. 64*box+63).  Key group g consumes tiles g, g+G, ... so the
// stage count is a multiple of G: each stage then always serves the same group,
// which waits for every fill of it in order (an mbarrier tells two successive
// phases apart only).
template <int HD, bool SPLIT, int HPC, int KT>
__global__ void __launch_bounds__(NTH, 2) attn_tma_kernel(const __grid_constant__ CUtensorMap tmK,
                                                       const __grid_constant__ CUtensorMap tmV, AttnTmaArgs a) {
    constexpr int PL = SPLIT ? 2 : 1;
    constexpr int NBOX = HD / 64;                     // boxes per K (or V) tile: 64 dims each
    constexpr int BOXB = PL * KT * 128;               // bytes of one box (all planes)
    constexpr int STAGE = 2 * NBOX * BOXB;            // K and V of one tile
    constexpr int G = NCW / HPC;                      // key groups
    constexpr int COMBINE = G * HPC * 16 * (HD + 2) * 4;  // key-group partials, staged in the ring
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int stages = a.stages;
    const int S = a.n_splits;
    const int pairs = HPC * 16, ppc = (pairs + S - 1) / S;  // (head, row) pairs; pairs per owner CTA
    const size_t ring_bytes = max((size_t)stages * STAGE, (size_t)COMBINE);
    float *recv_o = (float *)(ring + ring_bytes);              // [S][ppc][HD]
    float *recv_ml = recv_o + (size_t)S * ppc * HD;              // [S][ppc][2]
    uint64_t *full = (uint64_t *)(recv_ml + (size_t)S * ppc * 2);
    uint64_t *empty = full + stages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], HPC);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // every CTA of the cluster has started before any pushes into another's shared memory
    if (S > 1) cluster_arrive_relaxed();
    pdl_trigger();

    const int tile = blockIdx.x, hgrp = blockIdx.y, split = blockIdx.z;
    const int grp = a.nq / a.nkv;
    const int h0 = hgrp * HPC;             // first q head of the CTA
    const int kvh = h0 / grp;
    const int r0 = tile * a.rows_per_tile;
    const int nrows = min(a.rows_per_tile, a.R - r0);
    if (warp == NCW) {
        // While the projection before this kernel finishes: pull this CTA's K/V
        // tiles and the row metadata into L2.  The metadata read here (through
        // L2, no L1 line) may predate this pass; it only steers the prefetch.
        // The K/V rows the projection is still writing reach L2 after their
        // prefetch and replace it there, so the loads below see them.
        int nk_s = lane < nrows ? __ldcg(&a.meta[r0 + lane].nk) : 0;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) nk_s = max(nk_s, __shfl_xor_sync(0xffffffffu, nk_s, o2));
        const int seq_s = __ldcg(&a.meta[r0].seq);
        nk_s = min(max(nk_s, 0), a.max_len);
        if (seq_s >= 0 && seq_s < a.n_seq) {
            int p0, p1;
            split_range(nk_s, KT, S, split, p0, p1);
            const int sh = seq_s * a.nkv + kvh;
            // lane j: tile p0 + j / (2 * NBOX), box (j / 2) % NBOX, K (even j) or V (odd j)
            for (int j = lane; j < (p1 - p0) * 2 * NBOX; j += 32) {
                const int t = p0 + j / (2 * NBOX), b = (j / 2) % NBOX;
                tma_box_prefetch((j & 1) ? &tmV : &tmK, 64 * b, t * KT, sh, a.layer, SPLIT);
            }
        }
    }
    if (a.dep_ctr) {
        // q, K and V come from the projection before this kernel: wait until each of
        // its CTAs has signalled (acquire), then make its writes visible to TMA
        if (threadIdx.x == 0) {
            bool ok = true;
            const unsigned long long t0 = gtimer();
            while (ld_acquire_gpu(a.dep_ctr) < a.dep_target) {
                if (gtimer() - t0 > WAIT_NS) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
            if (!ok && a.err) atomicOr(a.err, 32);
            asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        __syncthreads();
    } else {
        __syncthreads();
        pdl_wait();  // q, K and V come from the projection before this kernel
    }

    // longest visible key range of the tile's rows (<= 16 rows), the same in every lane
    int nk_max = lane < nrows ? a.meta[r0 + lane].nk : 0;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) nk_max = max(nk_max, __shfl_xor_sync(0xffffffffu, nk_max, o2));
    const int seq = a.meta[r0].seq;
    int t0, t1;
    split_range(nk_max, KT, S, split, t0, t1);
    const int nt = t1 - t0;

    if (warp == NCW) {
        // ---------------- producer: one thread streams the split's tiles ----------------
        if (lane == 0) {
            const int sh = seq * a.nkv + kvh;
            for (int j = 0; j < nt; ++j) {
                const int s = j % stages;
                if (j >= stages && !mbar_wait(&empty[s], ((j / stages) - 1) & 1, a.err)) break;
                uint8_t *st = ring + (size_t)s * STAGE;
                mbar_expect_tx(&full[s], STAGE);
                const int key0 = (t0 + j) * KT;
#pragma unroll
                for (int b = 0; b < NBOX; ++b) {
                    tma_box(st + b * BOXB, &tmK, 64 * b, key0, sh, a.layer, SPLIT, &full[s]);
                    tma_box(st + (NBOX + b) * BOXB, &tmV, 64 * b, key0, sh, a.layer, SPLIT, &full[s]);
                }
            }
        }
    }

    // ---------------- consumers: warp = (key group g, head hw) ----------------
    const int hw = warp % HPC, g = warp / HPC;
    const int h = h0 + hw;
    const int ra = lane >> 2, rb = ra + 8;  // the two rows of this thread's accumulators
    float o[HD / 8][4];
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    if (warp < NCW) {
        const int nk_a = ra < nrows ? a.meta[r0 + ra].nk : 0;
        const int nk_b = rb < nrows ? a.meta[r0 + rb].nk : 0;
        // Q fragments (A operand, 16 rows x HD); ql: lo plane
        uint32_t qa[HD / 16][4], ql[SPLIT ? HD / 16 : 1][4];
        const bf16 *qa_row = a.q + (size_t)(r0 + ra) * a.ldq + h * HD;
        const bf16 *qb_row = a.q + (size_t)(r0 + rb) * a.ldq + h * HD;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
            const int c0 = kk * 16 + (lane & 3) * 2;
            qa[kk][0] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0) : 0u;
            qa[kk][1] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0) : 0u;
            qa[kk][2] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0 + 8) : 0u;
            qa[kk][3] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0 + 8) : 0u;
            if constexpr (SPLIT) {
                ql[kk][0] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + a.lo + c0) : 0u;
                ql[kk][1] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + a.lo + c0) : 0u;
                ql[kk][2] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + a.lo + c0 + 8) : 0u;
                ql[kk][3] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + a.lo + c0 + 8) : 0u;
            }
        }
        bool dead = false;  // a wait gave up: skip the remaining tiles without waiting again
#pragma unroll 1
        for (int j = g; j < nt; j += G) {
            const int s = j % stages;
            const bool ok = !dead && mbar_wait(&full[s], (j / stages) & 1, a.err);
            dead = !ok;
            const uint32_t st = smem_u32(ring + (size_t)s * STAGE);
            const int key0 = (t0 + j) * KT;
            // S = Q K^T over KT keys: KT/8 n-tiles of 8 keys
            float sc[KT / 8][4];
#pragma unroll
            for (int nt8 = 0; nt8 < KT / 8; ++nt8) sc[nt8][0] = sc[nt8][1] = sc[nt8][2] = sc[nt8][3] = 0.f;
            if (ok) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
                    for (int np = 0; np < KT / 16; ++np) {
                        // matrices (keys 0-7, d 0-7), (keys 0-7, d 8-15), (keys 8-15, d 0-7), (keys 8-15, d 8-15)
                        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
                        const uint32_t addr = st + (dim >> 6) * BOXB + swz(key, dim & 63);
                        uint32_t b0, b1, b2, b3;
                        ldm_x4(b0, b1, b2, b3, addr);
                        mma16816(sc[2 * np], qa[kk], b0, b1);
                        mma16816(sc[2 * np + 1], qa[kk], b2, b3);
                        if constexpr (SPLIT) {
                            mma16816(sc[2 * np], ql[kk], b0, b1);
                            mma16816(sc[2 * np + 1], ql[kk], b2, b3);
                            ldm_x4(b0, b1, b2, b3, addr + KT * 128);  // lo plane of the box
                            mma16816(sc[2 * np], qa[kk], b0, b1);
                            mma16816(sc[2 * np + 1], qa[kk], b2, b3);
                        }
                    }
                }
            }
            // mask + online softmax (log2 domain)
            float mx_a = m_a, mx_b = m_b;
#pragma unroll
            for (int nt8 = 0; nt8 < KT / 8; ++nt8) {
                const int key = key0 + nt8 * 8 + (lane & 3) * 2;
                sc[nt8][0] = ok && key < nk_a ? sc[nt8][0] * a.scale_log2 : -INFINITY;
                sc[nt8][1] = ok && key + 1 < nk_a ? sc[nt8][1] * a.scale_log2 : -INFINITY;
                sc[nt8][2] = ok && key < nk_b ? sc[nt8][2] * a.scale_log2 : -INFINITY;
                sc[nt8][3] = ok && key + 1 < nk_b ? sc[nt8][3] * a.scale_log2 : -INFINITY;
                mx_a = fmaxf(mx_a, fmaxf(sc[nt8][0], sc[nt8][1]));
                mx_b = fmaxf(mx_b, fmaxf(sc[nt8][2], sc[nt8][3]));
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
            for (int nt8 = 0; nt8 < KT / 8; ++nt8) {
                sc[nt8][0] = exp2f(sc[nt8][0] - ua);
                sc[nt8][1] = exp2f(sc[nt8][1] - ua);
                sc[nt8][2] = exp2f(sc[nt8][2] - ub);
                sc[nt8][3] = exp2f(sc[nt8][3] - ub);
                sa += sc[nt8][0] + sc[nt8][1];
                sb += sc[nt8][2] + sc[nt8][3];
            }
            l_a = l_a * ca + sa;
            l_b = l_b * cb + sb;
#pragma unroll
            for (int jj = 0; jj < HD / 8; ++jj) {
                o[jj][0] *= ca;
                o[jj][1] *= ca;
                o[jj][2] *= cb;
                o[jj][3] *= cb;
            }
            // O += P V : P as the A operand (KT/16 k-steps of 16 keys), V by transposed ldmatrix
            if (ok) {
                const uint32_t vst = st + NBOX * BOXB;
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk) {
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
                        const uint32_t addr = vst + (dim >> 6) * BOXB + swz(key, dim & 63);
                        uint32_t b0, b1, b2, b3;
                        ldm_x4_t(b0, b1, b2, b3, addr);
                        mma16816(o[2 * dp], pa, b0, b1);
                        mma16816(o[2 * dp + 1], pa, b2, b3);
                        if constexpr (SPLIT) {
                            mma16816(o[2 * dp], pl, b0, b1);
                            mma16816(o[2 * dp + 1], pl, b2, b3);
                            ldm_x4_t(b0, b1, b2, b3, addr + KT * 128);
                            mma16816(o[2 * dp], pa, b0, b1);
                            mma16816(o[2 * dp + 1], pa, b2, b3);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);  // the stage may be reloaded
        }
        // row sums across the quad
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    }

    // ---------------- merge the key groups of this CTA (G > 1) ----------------
    // every tile has been consumed (so no TMA write is in flight): the ring is free
    __syncthreads();
    float *cst_o = reinterpret_cast<float *>(ring);        // [G][HPC][16][HD]
    float *cst_ml = cst_o + (size_t)G * HPC * 16 * HD;     // [G][HPC][16][2]
    if (G > 1) {
        if (warp < NCW) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int row = half ? rb : ra;
                float *dst = cst_o + (((size_t)g * HPC + hw) * 16 + row) * HD + (lane & 3) * 2;
#pragma unroll
                for (int jj = 0; jj < HD / 8; ++jj)
                    *reinterpret_cast<float2 *>(dst + jj * 8) = make_float2(o[jj][2 * half], o[jj][2 * half + 1]);
                if ((lane & 3) == 0)
                    *reinterpret_cast<float2 *>(cst_ml + (((size_t)g * HPC + hw) * 16 + row) * 2) =
                        make_float2(half ? m_b : m_a, half ? l_b : l_a);
            }
        }
        __syncthreads();
    }
    // ---------------- push this CTA's partial of every (head, row) pair to its owner ----------------
    if (S > 1) cluster_wait();
    if (G > 1) {
        constexpr int D4 = HD / 4;
#pragma unroll 1
        for (int e = threadIdx.x; e < HPC * 16 * D4; e += NTH) {
            const int pair = e / D4, d0 = (e % D4) * 4;  // pair = head within CTA * 16 + row
            float mstar = -INFINITY;
#pragma unroll
            for (int gg = 0; gg < G; ++gg) mstar = fmaxf(mstar, cst_ml[((size_t)gg * HPC * 16 + pair) * 2]);
            const float mu = mstar == -INFINITY ? 0.f : mstar;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            float lsum = 0.f;
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                const float2 ml = *reinterpret_cast<const float2 *>(cst_ml + ((size_t)gg * HPC * 16 + pair) * 2);
                const float w = exp2f(ml.x - mu);
                const float4 v = *reinterpret_cast<const float4 *>(cst_o + ((size_t)gg * HPC * 16 + pair) * HD + d0);
                lsum += ml.y * w;
                acc.x += v.x * w;
                acc.y += v.y * w;
                acc.z += v.z * w;
                acc.w += v.w * w;
            }
            const int owner = pair / ppc, pl = pair - owner * ppc;
            float *dst = recv_o + ((size_t)split * ppc + pl) * HD + d0;
            if (S > 1) st_cluster_v4(dst, (uint32_t)owner, acc);
            else *reinterpret_cast<float4 *>(dst) = acc;
            if (d0 == 0) {
                float *dml = recv_ml + ((size_t)split * ppc + pl) * 2;
                if (S > 1) st_cluster_v2(dml, (uint32_t)owner, mstar, lsum);
                else *reinterpret_cast<float2 *>(dml) = make_float2(mstar, lsum);
            }
        }
    } else if (warp < NCW) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int row = half ? rb : ra;
            const int pair = hw * 16 + row, owner = pair / ppc, pl = pair - owner * ppc;
            float *dst = recv_o + ((size_t)split * ppc + pl) * HD + (lane & 3) * 2;
#pragma unroll
            for (int jj = 0; jj < HD / 8; ++jj) {
                if (S > 1) st_cluster_v2(dst + jj * 8, (uint32_t)owner, o[jj][2 * half], o[jj][2 * half + 1]);
                else *reinterpret_cast<float2 *>(dst + jj * 8) = make_float2(o[jj][2 * half], o[jj][2 * half + 1]);
            }
            if ((lane & 3) == 0) {
                float *dml = recv_ml + ((size_t)split * ppc + pl) * 2;
                if (S > 1) st_cluster_v2(dml, (uint32_t)owner, half ? m_b : m_a, half ? l_b : l_a);
                else *reinterpret_cast<float2 *>(dml) = make_float2(half ? m_b : m_a, half ? l_b : l_a);
            }
        }
    }
    if (S > 1) cluster_sync_all();  // every push is visible (release / acquire)
    else __syncthreads();

    // ---------------- owners: merge the splits' partials in split order, store ----------------
    const int p0 = split * ppc, p1 = min(pairs, p0 + ppc);
    constexpr int D4 = HD / 4;
#pragma unroll 1
    for (int e = threadIdx.x; e < (p1 - p0) * D4; e += NTH) {
        const int pl = e / D4, d0 = (e % D4) * 4;
        const int pair = p0 + pl, hh = pair / 16, row = pair % 16;
        if (row >= nrows) continue;
        float mstar = -INFINITY;
#pragma unroll 1
        for (int s2 = 0; s2 < S; ++s2) mstar = fmaxf(mstar, recv_ml[((size_t)s2 * ppc + pl) * 2]);
        const float mu = mstar == -INFINITY ? 0.f : mstar;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lsum = 0.f;
#pragma unroll 1
        for (int s2 = 0; s2 < S; ++s2) {
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
        bf16 *dst = a.out + (size_t)(r0 + row) * a.ldo + (h0 + hh) * HD + d0;
        store_pair(dst, a.lo, acc.x * inv, acc.y * inv);
        store_pair(dst + 2, a.lo, acc.z * inv, acc.w * inv);
    }
    if (a.done_ctr) {  // every writer fences (generic and async proxy) before the signal
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) atomicAdd(a.done_ctr, 1);
    }
}

}  // namespace atm

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

bool attn_tma_supported(int hd, int grp) { return (hd == 64 || hd == 128) && grp >= 1 && grp <= 8; }

bool attn_tma_make_map(CUtensorMap *map, const bf16 *cache, int hd, int max_len, int n_seq_heads, int n_layers,
                       size_t layer_elems, size_t lo, int kt) {
    auto enc = encode_fn();
    if (!enc || !cache) return false;
    memset(map, 0, sizeof *map);
    const cuuint32_t rank = lo ? 5 : 4;
    cuuint64_t dims[5] = {(cuuint64_t)hd, (cuuint64_t)max_len, (cuuint64_t)n_seq_heads, (cuuint64_t)n_layers, 2};
    cuuint64_t strides[4] = {(cuuint64_t)hd * 2, (cuuint64_t)max_len * hd * 2, (cuuint64_t)layer_elems * 2,
                             (cuuint64_t)lo * 2};
    cuuint32_t box[5] = {64, (cuuint32_t)kt, 1, 1, 2};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if ((lo * 2) % 16 || (layer_elems * 2) % 16) return false;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<bf16 *>(cache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q heads per CTA.  Measured on B200 (Qwen3-8B shape: 32 q heads, 8 kv heads,
// 16-row query tiles, ~530-key contexts; attention us per launch):
//  - one query tile (batch 1): one q head per CTA, 8 key splits (16.8; the GQA
//    group per CTA 18.8);
//  - up to 64 (tile, kv head) pairs (batch 4, 8): the GQA group of 4 heads per
//    CTA with the keys split to ~128 CTAs (batch 4: 37.3 -> 25.0, batch 8: 45.4
//    -> 35.2 against one head per CTA);
//  - more (batch 16, 32): 2 heads per CTA, no split (batch 16: 68.5 -> 51.3,
//    batch 32 with 4 heads per CTA: 133.6 -> 104.4).
// Fewer than 4 query tiles (one or two sequences, blocks up to 32 rows) and
// prefill chunks (the tiles of one sequence, causal) take one q head per CTA
// with the keys split to fill the GPU while the (tile, kv head) pairs do not
// fill it (block 32 at batch 1: 30.8 us against 33.2 us with the GQA group),
// 2 heads per CTA once they do (prefill, against the GQA group per CTA:
// 1024-token prompt 0.138 -> 0.071 s, 8192 tokens 0.625 -> 0.566 s).
static bool attn_tma_batched(int n_tiles, bool one_seq) { return !one_seq && n_tiles >= 4; }

int attn_tma_hpc(int grp, int n_tiles, int nkv, int num_sms, bool one_seq) {
    if (!attn_tma_batched(n_tiles, one_seq)) {
        if (n_tiles * nkv < num_sms) return 1;
        return grp % 2 == 0 ? 2 : 1;
    }
    if (n_tiles * nkv <= 64 && grp % 4 == 0) return 4;
    return grp % 2 == 0 ? 2 : 1;
}
// keys per tile: 16 when four key groups share the ring (its stages stay small),
// 32 for one group
int attn_tma_kt(int hpc) { return hpc == 4 ? 32 : 16; }

static size_t attn_tma_stage(int hd, bool split, int kt) { return (size_t)2 * (hd / 64) * (split ? 2 : 1) * kt * 128; }

// stages: a multiple of the key groups, as many as fit in ~100 KB (two CTAs per SM);
// rounds > 0: rounds x the key groups
static int attn_tma_stages(int hd, bool split, int hpc, int rounds) {
    const int G = atm::NCW / hpc;
    if (rounds > 0) return G * rounds;
    const size_t st = attn_tma_stage(hd, split, attn_tma_kt(hpc));
    const int k = std::max(1, (int)((100u << 10) / (st * G)));
    return G * std::min(k, std::max(1, 4 / G));
}

// Decomposition overrides for measurement sweeps (unset or 0 = the built-in
// policy): DFLASH_ATTN_HPC (q heads per CTA: 1, 2 or 4), DFLASH_ATTN_SPLITS (key
// splits, at most 8), DFLASH_ATTN_ROUNDS (ring stages per key group)
struct AttnTune {
    int hpc = 0, splits = 0, rounds = 0;
    AttnTune() {
        auto env_int = [](const char *name) {
            const char *v = getenv(name);
            return v ? atoi(v) : 0;
        };
        hpc = env_int("DFLASH_ATTN_HPC");
        splits = env_int("DFLASH_ATTN_SPLITS");
        rounds = std::max(0, std::min(16, env_int("DFLASH_ATTN_ROUNDS")));
    }
};
static const AttnTune &attn_tune() {
    static const AttnTune t;
    return t;
}

static size_t attn_tma_smem(int hd, bool split, int hpc, int S, int stages) {
    const size_t stage = attn_tma_stage(hd, split, attn_tma_kt(hpc));
    const int G = atm::NCW / hpc;
    const size_t combine = (size_t)G * hpc * 16 * (hd + 2) * 4;
    const size_t ring = std::max((size_t)stages * stage, combine);
    const int ppc = (hpc * 16 + S - 1) / S;
    return 1024 + ring + (size_t)S * ppc * (hd + 2) * 4 + (size_t)2 * stages * 8 + 64;
}

template <int HD, bool SPLIT, int HPC>
static cudaError_t launch_one(const CUtensorMap &mk, const CUtensorMap &mv, const AttnTmaArgs &a, int n_tiles,
                              cudaStream_t s) {
    constexpr int KT = HPC == 4 ? 32 : 16;
    auto kern = atm::attn_tma_kernel<HD, SPLIT, HPC, KT>;
    ensure_smem_attr((const void *)kern);
    const size_t smem = attn_tma_smem(HD, SPLIT, HPC, a.n_splits, a.stages);
    return launch_k(kern, dim3(n_tiles, a.nq / HPC, a.n_splits), dim3(atm::NTH), smem, s, a.n_splits, mk, mv, a);
}

int launch_attention_tma(const AttnTmaMaps &maps, AttnTmaArgs a, int hd, bool split, int num_sms, cudaStream_t s) {
    if (a.R <= 0) return 0;
    const int grp = a.nq / a.nkv;
    const int n_tiles = (a.R + a.rows_per_tile - 1) / a.rows_per_tile;
    const AttnTune &tune = attn_tune();
    int hpc = attn_tma_hpc(grp, n_tiles, a.nkv, num_sms, a.one_seq != 0);
    if ((tune.hpc == 1 || tune.hpc == 2 || tune.hpc == 4) && grp % tune.hpc == 0) hpc = tune.hpc;
    const int kt = attn_tma_kt(hpc);
    const CUtensorMap &mk = kt == 32 ? maps.k32 : maps.k16, &mv = kt == 32 ? maps.v32 : maps.v16;
    const int units = n_tiles * (a.nq / hpc);
    // splits of one (tile, head group) form a cluster of at most 8 CTAs; no more
    // splits than key tiles the longest context has.  Batched decode (the
    // measurements above): ~128 CTAs for the 4-head form, no split for 2 heads;
    // otherwise enough CTAs for two per SM
    const bool batched = attn_tma_batched(n_tiles, a.one_seq != 0) && hpc != 1;
    const int want = !batched ? (2 * num_sms + units - 1) / units : hpc == 4 ? 128 / units : 1;
    a.n_splits = std::max(1, std::min({8, want, (a.max_len + kt - 1) / kt}));
    if (tune.splits > 0) a.n_splits = std::min({8, tune.splits, (a.max_len + kt - 1) / kt});
    a.stages = attn_tma_stages(hd, split, hpc, tune.rounds);
    cudaError_t e = cudaErrorInvalidValue;
#define ATM_CASE(HD_, SP_, HPC_)                                                  \
    if (hd == HD_ && split == SP_ && hpc == HPC_) e = launch_one<HD_, SP_, HPC_>(mk, mv, a, n_tiles, s);
    ATM_CASE(128, true, 1) ATM_CASE(128, true, 2) ATM_CASE(128, true, 4)
    ATM_CASE(128, false, 1) ATM_CASE(128, false, 2) ATM_CASE(128, false, 4)
    ATM_CASE(64, true, 1) ATM_CASE(64, true, 2) ATM_CASE(64, true, 4)
    ATM_CASE(64, false, 1) ATM_CASE(64, false, 2) ATM_CASE(64, false, 4)
#undef ATM_CASE
    if (e != cudaSuccess) return -1;
    return n_tiles * (a.nq / hpc) * a.n_splits;
}

}  // namespace dfl
