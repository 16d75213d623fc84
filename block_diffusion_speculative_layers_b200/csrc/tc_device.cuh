// tc_device.cuh -- device helpers shared by the tensor-core projection kernels:
// mbarriers, TMA tile loads, tcgen05 descriptors/MMA/TMEM loads, cluster
// helpers and the fused projection epilogues.
#pragma once

#include <cudaTypedefs.h>

#include "gemm_tc.h"

namespace dfl {
namespace tc {

constexpr int BK = 64;                 // bf16 K elements per stage = one 128-byte swizzle row
constexpr int A_BYTES = 128 * BK * 2;  // 16 KB weight tile per stage
constexpr int F8_A_BYTES = 128 * 128;  // FP8 weights: 128 rows x 128 codes per stage
constexpr int F8_PLANES = 4;           // FP8 weights: E4M3 planes per activation value (MX block scales)

// tensor-memory columns to allocate for n used columns: a power of two >= 32
__host__ __device__ constexpr int tmem_cols_for(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512; }
constexpr int NT = 192;
constexpr int CH = 16;                 // accumulator columns per epilogue chunk
constexpr int STG_LD = CH + 1;
constexpr unsigned long long WAIT_NS = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
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

// Bounded wait: false (and error bit 4) after WAIT_NS.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, int *err) {
    if (mbar_try(b, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try(b, parity)) return true;
        if (gtimer() - t0 > WAIT_NS) {
            if (err) atomicOr(err, 4);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// L2 policy for streamed weights: each weight byte is read once per decode
// pass, so it is marked evict-first and does not push activations, K/V, the
// per-row norm statistics or the kernels' own code out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// L2 prefetch of one weight box (no shared memory, no completion): a later TMA
// load of the same box then hits L2 instead of HBM
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

// weight tile load with an L2 cache-policy hint
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
        "%4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

// Two-plane activation tile: box {BK, rows, 2} of a 3-D map whose third
// dimension steps from the hi plane to the lo plane; lands as [2][rows][BK].
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// K-major operand, 128-byte swizzle: 8-row groups 1024 B apart (SBO), sm100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;               // leading byte offset (16 B; unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;     // stride byte offset
    d |= (uint64_t)1 << 46;               // descriptor version
    d |= (uint64_t)2 << 61;               // SWIZZLE_128B
    return d;
}

// bf16 x bf16 -> fp32, A and B K-major, M = 128, N = tm.
__host__ __device__ constexpr uint32_t idesc_bf16(int tm) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(tm >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Columns c..c+15 of a tile accumulator.  With a wide two-plane MMA (one
// N = 2*TM product over the hi and lo activation rows) the lo-plane partial
// sums sit lo_col = TM columns further on and are added here; lo_col = 0 otherwise.
__device__ __forceinline__ void acc_ld16(uint32_t taddr, int c, int lo_col, float *v) {
    tmem_ld16(taddr + (uint32_t)c, v);
    if (lo_col) {
        float t[16];
        tmem_ld16(taddr + (uint32_t)(lo_col + c), t);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += t[j];
    }
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *p >= target.  false (error bit 8) after WAIT_NS.
__device__ __forceinline__ bool wait_counter(const int *p, int target, int *err) {
    if (ld_acquire(p) >= target) return true;
    const unsigned long long t0 = gtimer();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (ld_acquire(p) >= target) return true;
        if (gtimer() - t0 > WAIT_NS) {
            if (err) atomicOr(err, 8);
            return false;
        }
        __nanosleep(32);
    }
}

// Wait for the producer of this kernel's inputs: with a completion counter
// (dep != nullptr), until every CTA of the previous kernel has signalled
// (acquire; then TMA reads see its writes); otherwise griddepcontrol.wait.
__device__ __forceinline__ void dep_wait(const int *dep, int target, int *err) {
    if (dep) {
        wait_counter(dep, target, err);
        fence_proxy_async_global();
    } else {
        pdl_wait();
    }
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// ---------------------------------------------------------------------------
// fused epilogue on one chunk of up to CH accumulator columns (activation rows
// m0c .. m0c+nc-1) for weight row n_local of the tile.  Global loads of a
// chunk are issued together before any use.
// ---------------------------------------------------------------------------
// Per-row RMSNorm scales of a tile's rows m_base .. m_base+rows-1 (folded
// norm): 8 epilogue threads per row each sum every 8th per-tile sum of squares
// (all loads issued together), combined by shuffles in a fixed order.  Runs
// once per tile, before the accumulator is ready; the 128 epilogue threads
// (64..191) all take part.
constexpr int RS_MAX = 256;  // rows of one tile (TM <= 256)
__device__ __forceinline__ void all_row_scales(const Epi<bf16> &e, int m_base, int rows, int M, float *rs) {
    epi_bar();  // the previous tile's epilogue may still read rs
    const int t = (int)threadIdx.x - 64;
    const int part = t & 7, rr = t >> 3;
    for (int r0 = 0; r0 < rows; r0 += 16) {
        const int r = r0 + rr, m = m_base + r;
        float a = 0.f;
        if (r < rows && m < M) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int tile = part + 8 * u;
                v[u] = tile < e.rs_tiles ? e.rs_ssq[(size_t)tile * e.rs_ld + m] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) a += v[u];
            for (int tile = part + 64; tile < e.rs_tiles; tile += 8) a += e.rs_ssq[(size_t)tile * e.rs_ld + m];
        }
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        if (part == 0 && r < rows) rs[r] = 1.0f / sqrtf(a * e.rs_inv_n + e.rs_eps);
    }
    epi_bar();
}

// y -> bf16(y * g_next) and the tile's per-row sum of squares (fixed reduction order).
template <int W>
__device__ __forceinline__ void norm_outputs(const TcParams &p, const Epi<bf16> &e, int nt, int n, int q, int lane,
                                             int m0c, int nc, const float *y, float2 *red, const float *gn_pre) {
    const int M = p.M;
    const bool nok = n < p.N;
    const float gn = gn_pre ? *gn_pre : ((nok && e.g_next) ? e.g_next[n] : 0.f);
#pragma unroll
    for (int j = 0; j < W; ++j) {
        const bool ok = nok && j < nc && m0c + j < M;
        if (ok && e.xg) st_act(e.xg, (size_t)(m0c + j) * e.xg_ld + n, e.lo, y[j] * gn);
        float sq = ok ? y[j] * y[j] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) red[q * CH + j].x = sq;
    }
    epi_bar();
    if (threadIdx.x >= 64 && threadIdx.x < 64 + W) {
        const int j = threadIdx.x - 64, m = m0c + j;
        if (j < nc && m < M && e.ssq_out)
            e.ssq_out[(size_t)nt * e.ssq_ld + m] = (red[j].x + red[CH + j].x) + (red[2 * CH + j].x + red[3 * CH + j].x);
    }
    epi_bar();
}

// Row metadata of a QKV chunk's columns (activation rows m0c..m0c+nc-1) into
// smeta[]: aux = 0 block row, 1 context row whose K/V is written, -1 skip.
__device__ __forceinline__ void qkv_fill_meta(const Epi<bf16> &e, int m0c, int nc, int M, RowMeta *smeta) {
    if (threadIdx.x >= 64 && threadIdx.x < 64 + CH) {
        const int j = threadIdx.x - 64, m = m0c + j;
        RowMeta mt;
        mt.seq = mt.pos = mt.nk = 0;
        mt.aux = -1;  // -1: skip this column
        if (j < nc && m < M) {
            if (m >= e.R_blk) {
                mt = e.ctx_meta[m - e.R_blk];
                mt.aux = mt.aux ? 1 : -1;
            } else {
                mt = e.meta[m];
                mt.aux = 0;
            }
        }
        smeta[j] = mt;
    }
    epi_bar();
}

// RoPE (cos, sin) of this thread's weight row for each column of the chunk.
template <int W>
__device__ __forceinline__ void qkv_rope_factors(const Epi<bf16> &e, int cg, int N_ok, const RowMeta *smeta,
                                                 float2 *cs) {
    const int hd = e.hd, half = hd >> 1, qd = e.nq * hd, kd = e.nkv * hd;
    const int d = cg % hd;
    const int i = d < half ? d : d - half;
    const bool rot = N_ok && cg < qd + kd;  // q and k rows are rotated
#pragma unroll
    for (int j = 0; j < W; ++j)
        cs[j] = rot && smeta[j].aux >= 0 ? e.rope[(size_t)smeta[j].pos * half + i] : make_float2(1.f, 0.f);
}

// Inputs of a chunk's fused epilogue that do not depend on the accumulator
// (residual rows, tap rows, the next norm's gain; QKV row metadata and RoPE
// factors).  They are loaded while the mainloop still streams, so that after
// the last MMA the epilogue only computes and stores -- loads issued then would
// queue behind the next projection's weight prefetch.
struct EpiIn {
    float xo[CH];
    int trow[CH];
    float gn;
    float2 cs[CH];
};

template <int KIND, int W>
__device__ __forceinline__ void epi_prefetch(const TcParams &p, const Epi<bf16> &e, int nt, int n_local, int m0c,
                                             int nc, EpiIn &in, RowMeta *smeta) {
    const int M = p.M;
    const int n = nt * 128 + n_local;
    const bool nok = n < p.N;
    if (KIND == EPI_RESID || KIND == EPI_NORMOUT) {
        in.gn = (nok && e.g_next) ? e.g_next[n] : 0.f;
        if (KIND == EPI_RESID) {
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const bool ok = nok && j < nc && m0c + j < M;
                in.xo[j] = ok ? e.x[(size_t)(m0c + j) * p.N + n] : 0.f;
                in.trow[j] = (ok && e.taps.n) ? e.meta[m0c + j].aux : 0;
            }
        }
    } else if (KIND == EPI_QKV) {
        qkv_fill_meta(e, m0c, nc, M, smeta);
        qkv_rope_factors<W>(e, e.col0 + n, nok, smeta, in.cs);
    }
}

// W: columns the chunk can hold (4, 8 or 16).  The epilogue runs once per CTA
// and launch, so its code is fetched cold each time; K-split CTAs finishing only
// a few columns use a narrow instantiation to keep that code short.
template <int KIND, int W = CH>
__device__ __forceinline__ void epilogue_chunk(const TcParams &p, const Epi<bf16> &e, int nt, int n_local, int q,
                                               int lane, int m0c, int nc, const float *vin, float *stg, float2 *red,
                                               RowMeta *smeta, const float *rs, const EpiIn *pre = nullptr) {
    // rs[j]: RMSNorm scale of row m0c + j (folded norm; see all_row_scales);
    // pre: this chunk's inputs loaded by epi_prefetch (nullptr: load them here)
    const int M = p.M;
    float v[CH];
    if (KIND == EPI_QKV || KIND == EPI_SWIGLU || KIND == EPI_LOGITS || KIND == EPI_STORE) {
        if (e.rs_ssq) {
#pragma unroll
            for (int j = 0; j < W; ++j) v[j] = vin[j] * rs[j];
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) v[j] = vin[j];
        }
    } else {
#pragma unroll
        for (int j = 0; j < W; ++j) v[j] = vin[j];
    }
    if (KIND == EPI_STORE) {
        const int n = nt * 128 + n_local;
        if (n < p.N) {
#pragma unroll
            for (int j = 0; j < W; ++j)
                if (j < nc && m0c + j < M)
                    e.Y[(size_t)(e.row_map ? e.row_map[m0c + j] : m0c + j) * e.ldy + n] = v[j];
        }
    } else if (KIND == EPI_RESID) {
        const int n = nt * 128 + n_local;
        const bool nok = n < p.N;
        float xo[CH];
        int trow[CH];
        if (pre) {
#pragma unroll
            for (int j = 0; j < W; ++j) {
                xo[j] = pre->xo[j];
                trow[j] = pre->trow[j];
            }
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const bool ok = nok && j < nc && m0c + j < M;
                xo[j] = ok ? e.x[(size_t)(m0c + j) * p.N + n] : 0.f;
                trow[j] = (ok && e.taps.n) ? e.meta[m0c + j].aux : 0;
            }
        }
#pragma unroll
        for (int j = 0; j < W; ++j) {
            if (!(nok && j < nc && m0c + j < M)) continue;
            const float nx = xo[j] + v[j];
            xo[j] = nx;
            e.x[(size_t)(m0c + j) * p.N + n] = nx;
            for (int t = 0; t < e.taps.n; ++t)
                st_act(e.taps.base, (size_t)trow[j] * e.taps.ld + e.taps.col[t] + n, e.lo, nx);
        }
        if (e.ssq_out) norm_outputs<W>(p, e, nt, n, q, lane, m0c, nc, xo, red, pre ? &pre->gn : nullptr);
    } else if (KIND == EPI_NORMOUT) {
        norm_outputs<W>(p, e, nt, nt * 128 + n_local, q, lane, m0c, nc, v, red, pre ? &pre->gn : nullptr);
    } else if (KIND == EPI_LOGITS) {
        const int n = nt * 128 + n_local;
        const bool ok = n < p.N;
        bool bad = false;  // a non-finite logit anywhere in the row makes the argmax meaningless
#pragma unroll
        for (int j = 0; j < W; ++j) {
            const int m = m0c + j;
            const bool col = j < nc && m < M;
            bad |= ok && col && !isfinite(v[j]);
            if (p.keep_logits && ok && col) e.Y[(size_t)m * e.ldy + n] = v[j];
            float bv = (ok && col) ? v[j] : -INFINITY;
            int bi = (ok && col) ? n : 0x7fffffff;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
                const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
                argmax_merge(bv, bi, v2, i2);
            }
            if (lane == 0) red[q * CH + j] = make_float2(bv, __int_as_float(bi));
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0 && p.err) atomicOr(p.err, 1);
        epi_bar();
        if (threadIdx.x >= 64 && threadIdx.x < 64 + W) {
            const int j = threadIdx.x - 64;
            const int m = m0c + j;
            float bv = red[j].x;
            int bi = __float_as_int(red[j].y);
            for (int qq = 1; qq < 4; ++qq) argmax_merge(bv, bi, red[qq * CH + j].x, __float_as_int(red[qq * CH + j].y));
            if (j < nc && m < M) p.lm_part[(size_t)nt * p.M + m] = make_float2(bv, __int_as_float(bi));
        }
        epi_bar();
    } else if (KIND == EPI_SWIGLU) {
#pragma unroll
        for (int j = 0; j < W; ++j) stg[n_local * STG_LD + j] = v[j];
        epi_bar();
        if (n_local < 64) {
            const int f = nt * 64 + n_local;
            if (f < p.swiglu_F) {
#pragma unroll
                for (int j = 0; j < W; ++j) {
                    const int m = m0c + j;
                    if (j >= nc || m >= M) break;
                    const float up = stg[(n_local + 64) * STG_LD + j];
                    st_act(e.h, (size_t)m * p.swiglu_F + f, e.lo, silu_f(v[j]) * up);
                }
            }
        }
        epi_bar();
    } else if (KIND == EPI_QKV) {
        const int hd = e.hd, half = hd >> 1;
        const int qd = e.nq * hd, kd = e.nkv * hd;
        const int cg = e.col0 + nt * 128 + n_local;  // row of [Wq; Wk; Wv]
        if (e.qn_g) {
            // QK-norm: each q / k head (hd rows of this tile, tiles start on head
            // boundaries) is RMS-normalised per column before RoPE; per-warp sums of
            // squares over 32 rows, then over the head's warps in a fixed order
            const bool normed = nt * 128 + n_local < p.N && cg < qd + kd;
#pragma unroll
            for (int j = 0; j < W; ++j) {
                float sq = normed ? v[j] * v[j] : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                if (lane == 0) red[q * CH + j].x = sq;
            }
            epi_bar();
            const int w0 = (n_local / hd) * hd / 32, nw = hd / 32;
            const float g = normed ? (cg < qd ? e.qn_g[cg % hd] : e.kn_g[cg % hd]) : 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) {
                float a = 0.f;
                for (int w = 0; w < nw; ++w) a += red[(w0 + w) * CH + j].x;
                if (normed) v[j] *= g / sqrtf(a / (float)hd + e.qk_eps);
            }
            epi_bar();  // red is reused below
        }
#pragma unroll
        for (int j = 0; j < W; ++j) stg[n_local * STG_LD + j] = v[j];
        if (pre) epi_bar();  // smeta is already filled; stg must be complete before partners are read
        else qkv_fill_meta(e, m0c, nc, M, smeta);
        if (nt * 128 + n_local < p.N) {
            const int head_base = (cg / hd) * hd;
            const int d = cg - head_base;
            const int partner = n_local + (d < half ? half : -half);
            const bool is_q = cg < qd, is_k = !is_q && cg < qd + kd;
            float2 cs[CH];
            if (pre) {
#pragma unroll
                for (int j = 0; j < W; ++j) cs[j] = pre->cs[j];
            } else {
                qkv_rope_factors<W>(e, cg, true, smeta, cs);
            }
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const RowMeta mt = smeta[j];
                if (mt.aux < 0) continue;          // padding column or uncommitted context row
                const bool ctx = mt.aux == 1;
                if (ctx && is_q) continue;         // context rows only feed K/V
                float out = v[j];
                if (is_q || is_k) {
                    const float other = stg[partner * STG_LD + j];
                    out = d < half ? v[j] * cs[j].x - other * cs[j].y : v[j] * cs[j].x + other * cs[j].y;
                }
                if (is_q) {
                    st_act(e.q_out, (size_t)(m0c + j) * qd + cg, e.lo, out);
                } else {
                    const int hh = is_k ? (cg - qd) / hd : (cg - qd - kd) / hd;
                    bf16 *dst = (is_k ? e.kc : e.vc) + (((size_t)mt.seq * e.nkv + hh) * e.max_len + mt.pos) * hd;
                    st_act(dst, (size_t)d, e.lo, out);
                }
            }
        }
        epi_bar();
    }
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

// store v to the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ void st_cluster_f32(float *local, uint32_t rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// store 4 floats (16-byte aligned) to the same shared-memory location in CTA `rank`
__device__ __forceinline__ void st_cluster_v4(float *local, uint32_t rank, float a, float b, float c, float d) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// columns of a K-split tile finished by each CTA of the cluster (a multiple of 4)
__host__ __device__ constexpr int split_cols(int tm, int s) { return ((tm + s - 1) / s + 3) / 4 * 4; }

// generic address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ const float *peer_ptr(const float *p, uint32_t rank) {
    uint64_t out;
    asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const float *>(out);
}

}  // namespace tc
}  // namespace dfl
