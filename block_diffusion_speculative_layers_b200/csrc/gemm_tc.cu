// gemm_tc.cu -- tensor-core weight-streaming projection for bf16 models on
// sm_100a: TMA (SWIZZLE_128B) -> shared-memory ring -> tcgen05.mma (accumulator
// in TMEM) -> fused epilogue.
//
// Roles per CTA (192 threads):
//   warp 0      one thread issues TMA loads of the weight tile (two 64-row
//               boxes) and the activation tile into a ring of stages;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128 weight
//               rows, N=TM activation rows, or N=2*TM over both planes of
//               two-plane activations; K=16) and commits each consumed stage
//               back to the producer;
//   warps 2..5  epilogue: row scales of the folded RMSNorm and the inputs of
//               the fused epilogue are loaded while the main loop runs; then
//               tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31 = weight rows), the split-K exchange when the K
//               range is split, and the fused epilogue (store / RoPE + KV write
//               / residual + taps + next-norm inputs / SwiGLU / per-tile argmax).
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA
// records an error bit and drains.
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <type_traits>
#include <cstdio>
#include <cstring>

#include "gemm_tc.h"
#include "launch.h"

#include "tc_device.cuh"

namespace dfl {
namespace tc {

// Work split.  The host launches one CTA per (weight tile, activation-row
// tile).  Projections with fewer tiles than two per SM split the K range over
// a thread-block cluster of p.splits CTAs along z: each CTA accumulates its K
// range in TMEM and pushes the columns other CTAs finish into their shared
// memory; after one cluster barrier each CTA sums its columns over the cluster
// in rank order (identical results run to run) and runs the fused epilogue on
// them.  CTAs of ~110 KB leave room for the next kernel's CTA on the same SM,
// which starts streaming its weights early (programmatic dependent launch:
// weights are loaded before griddepcontrol.wait, activations after it).
// A 1-D grid smaller than the tile count makes CTAs loop over tiles with two
// TMEM accumulators (the epilogue of one tile overlapping the MMAs of the
// next); the host policy does not use that form at present.
// FP8 weights (F8): the weight tile arrives as E4M3 codes, 128 rows x 128 K
// (16 KB, one TMA box per 64 rows), half the bytes of bf16, and goes to the
// tensor cores as it is: tcgen05.mma kind::mxf8f6f4 with block scales.  The
// activations reach the kernel already in the MX block-scaled form: a small
// kernel before each FP8 projection (mx_quantize_kernel) rewrites the bf16
// rows (both planes) as F8_PLANES E4M3 planes with one power-of-two (UE8M0)
// scale per 32 values of a row and plane; plane p holds what planes 0..p-1
// left over, so the planes sum to the value within 2^-16 of its block's
// largest magnitude.  Each stage loads the planes of its 128 K by TMA (the N
// operand, N = F8_PLANES * TM) and their scale words; the epilogue warps copy
// the words into tensor memory (tcgen05.st) during the main loop.  The weight
// rows' block scales are all 1; each weight row's fp32 scale multiplies the
// plane-summed accumulator in the epilogue.

// Smallest E with m * 2^-E <= 448 (the largest E4M3 magnitude) for m > 0,
// kept inside [-126, 126]; 0 for m == 0.  m = 1.f * 2^x: E = x - 8 unless the
// fraction is above 0.75 (then m / 2^(x-8) would pass 448).
__device__ __forceinline__ int mx_exp(float m) {
    const uint32_t b = __float_as_uint(m);
    const int e = (int)(b >> 23) - 135 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return m > 0.f ? min(126, max(-126, e)) : 0;
}

// MX planes of 16 values, half of a 32-value block whose other half sits in
// lane ^ 1.  Plane p: E = mx_exp(block max of what is left), codes of
// left * 2^-E rounded to nearest E4M3 (never saturating: |left * 2^-E| <= 448),
// then left -= code * 2^E, which is exact.  code[p] holds the 16 codes in
// order (two per 16-bit half, the first in the low byte), ex[p] the exponent.
template <int P>
__device__ __forceinline__ void mx_planes16(float (&r)[16], uint4 (&code)[P], int (&ex)[P]) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(r[i]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        const int E = mx_exp(m);
        ex[p] = E;
        const float inv = __uint_as_float((uint32_t)(127 - E) << 23), sc = __uint_as_float((uint32_t)(127 + E) << 23);
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const __nv_fp8x2_storage_t c2 =
                __nv_cvt_float2_to_fp8x2(make_float2(r[2 * q] * inv, r[2 * q + 1] * inv), __NV_SATFINITE, __NV_E4M3);
            const float2 d = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(c2, __NV_E4M3)));
            r[2 * q] -= d.x * sc;
            r[2 * q + 1] -= d.y * sc;
            if (q & 1) w[q >> 1] |= (uint32_t)c2 << 16;
            else w[q >> 1] = (uint32_t)c2;
        }
        code[p] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// E4M3 x E4M3 -> fp32 with UE8M0 block scales from tensor memory (one per 32 K
// of each A row and B column), M = 128, K = 32
__device__ __forceinline__ void mma_mx(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
}

// Instruction descriptor of mma_mx: E4M3 A and B, both K-major, UE8M0 scales,
// M = 128, N = n; scale byte `kb` of the A and B scale words (the 32-K block
// within a 128-K stage).
__host__ __device__ constexpr uint32_t idesc_mx(int n, int kb) {
    return ((uint32_t)kb << 4) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(128 >> 4) << 24) |
           ((uint32_t)kb << 29);
}

// Plain (untiled) bulk copy global -> shared of `bytes` (a multiple of 16; both
// addresses 16-byte aligned), completing on mbarrier `bar`
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t a) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(a) : "memory");
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// The kernel body.  p and e are the launch's parameters (ungrouped launches
// read them in place, without a copy) or a grouped CTA's adjusted copies.
template <int TM, int KIND, bool F8, bool GR>
__device__ __forceinline__ void gemm_tc_body(const CUtensorMap &tmW, const CUtensorMap &tmX, const CUtensorMap &tmS,
                                             const TcParams &p, const Epi<bf16> &e, int stages, int g_row0,
                                             int g_wrow0) {
    constexpr bool grouped = GR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // bf16: the activation tile(s) of 64 K; F8: the activation planes of 128 K
    const int B_BYTES = F8 ? F8_PLANES * TM * 128 : TM * 128 * p.planes;
    const int A_ST = F8 ? F8_A_BYTES : A_BYTES, B_ST = B_BYTES;
    constexpr int SW_ST = F8 ? F8_PLANES * TM * 4 : 0;  // F8: scale words of a stage, [plane][row]
    // two planes and TM <= 128: one MMA with N = 2*TM covers the hi and lo rows
    // (they are contiguous in the stage), accumulating into 2*TM columns
    const bool wide = !F8 && p.planes == 2 && TM <= 128;
    const int lo_col = wide ? TM : 0;
    // F8: N = F8_PLANES * TM quantised rows (plane-major)
    const int NC1 = max(32, F8 ? F8_PLANES * TM : wide ? 2 * TM : TM);  // TMEM columns of one accumulator
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)stages * A_ST;
    uint32_t *sW = (uint32_t *)(sB + (size_t)stages * B_ST);  // F8: [stages] scale words
    // FP4 weights: [stages][128] exponent words of the stage's weight rows
    const bool f4 = F8 && p.w_bexp != nullptr;
    uint32_t *sE = (uint32_t *)((uint8_t *)sW + (size_t)stages * SW_ST);
    float *stg = (float *)((uint8_t *)sE + (f4 ? (size_t)stages * 512 : 0));
    float2 *red = (float2 *)(stg + 128 * STG_LD);
    RowMeta *smeta = (RowMeta *)(red + 4 * CH);
    float *rsc = (float *)(smeta + CH);       // [RS_MAX] row scales of the folded norm
    uint64_t *full = (uint64_t *)(rsc + RS_MAX);
    uint64_t *empty = full + stages;
    uint64_t *acc_full = empty + stages;   // [2]
    uint64_t *acc_empty = acc_full + 2;    // [2]
    uint64_t *sf_full = acc_empty + 2;  // F8: [stages] a stage's scale words are in tensor memory
    uint32_t *tmem_slot = (uint32_t *)(sf_full + (F8 ? stages : 0));
    // split-K receive buffer [S][128][cpr] (16-byte aligned, after the fixed area)
    float *recv = (float *)(((uintptr_t)(tmem_slot + 4) + 15) & ~(uintptr_t)15);
    EpiIn pre;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.splits;
    const bool split = S > 1;
    const int n_tiles_total = grouped ? p.n_tiles : p.n_tiles * p.m_tiles;
    // one tile per CTA: (blockIdx.x, blockIdx.y); a persistent launch would pass
    // a 1-D grid smaller than the tile count and stride over the tiles; a grouped
    // launch has one weight tile (blockIdx.x) of one expert's rows per CTA
    const bool persistent = !F8 && !split && !grouped && gridDim.y == 1 && (int)gridDim.x < n_tiles_total;
    const int tile0 = persistent || grouped ? blockIdx.x : blockIdx.y * p.n_tiles + blockIdx.x;
    const int tstride = persistent ? gridDim.x : n_tiles_total;
    const int k_per = (p.k_steps + S - 1) / S;
    const int kb = split ? blockIdx.z * k_per : 0;
    const int ke = split ? min(p.k_steps, kb + k_per) : p.k_steps;
    const int nk = max(0, ke - kb);
    // F8: after the accumulator, the weights' scale words (4 columns: row m at
    // lane m, column m / 32) and one 4-column group per stage (plane row n at
    // lane n % 32 of every lane quarter, column n / 32; byte b of a word = the
    // scale of 32-K block b of the stage), as measured on the device
    // FP4 weights: one 4-column group per stage for the weights' block scales too
    const int sf_cols = F8 ? (f4 ? 8 * stages : 4 + 4 * stages) : 0;
    const int ncols = tmem_cols_for((persistent ? 2 * NC1 : NC1) + sf_cols);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], F8 ? 5 : 1);  // F8: the four scale-copy warps + the MMA commit
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        mbar_init(&acc_empty[0], 4);
        mbar_init(&acc_empty[1], 4);
        if (F8)
            for (int s = 0; s < stages; ++s) mbar_init(&sf_full[s], 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    // F8 scale columns: the weights' (FP8: one group of constant 1.0 bytes; FP4: one
    // group per stage), then one group per stage for the activation planes
    const uint32_t tmem_sfa = tmem + (uint32_t)NC1, tmem_sfb = tmem_sfa + (f4 ? 4u * (uint32_t)stages : 4u);
    // K split: every CTA of the cluster has started before any pushes into another's
    // shared memory (arrive now; the epilogue warps wait before their first push)
    if (split) cluster_arrive_relaxed();
    pdl_trigger();

    // F8: copy every stage's activation scale words into tensor memory (warps
    // 2..5; lane i of warp w writes plane rows i, 32 + i, ... of lane quarter
    // w % 4, each quarter of the MMA reading its own copy)
    auto copy_scales = [&] {
        const int q = warp & 3;
        const uint32_t quarter = (uint32_t)(q * 32) << 16;
        // FP8: the weights' block scales are 1.0 (UE8M0 127) in every byte.  FP4:
        // A row 32q + lane of the stage takes its exponent word (loaded with the
        // stage) at lane 32q + lane, column q of the stage's group
        if (!f4) tmem_st4(tmem_sfa + quarter, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        bool dead = false;
        for (int kk = 0; kk < nk; ++kk) {
            const int s = kk % stages;
            if (!dead && !mbar_wait(&full[s], (kk / stages) & 1, p.err)) dead = true;
            const uint32_t *w = sW + (size_t)s * (F8_PLANES * TM);
            uint32_t w4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) w4[c] = (!dead && 32 * c + lane < F8_PLANES * TM) ? w[32 * c + lane] : 0x7F7F7F7Fu;
            if (f4) tmem_st1(tmem_sfa + (uint32_t)(s * 4 + q) + quarter, dead ? 0x7F7F7F7Fu : sE[s * 128 + q * 32 + lane]);
            tmem_st4(tmem_sfb + (uint32_t)(s * 4) + quarter, w4[0], w4[1], w4[2], w4[3]);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sf_full[s]);
                mbar_arrive(&empty[s]);
            }
        }
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer: one continuous ring over all tiles of this CTA ----------------
            const uint64_t wpol = l2_evict_first_policy();
            const int kstep = F8 ? 2 * BK : BK;  // K elements per stage
            auto load_x = [&](int s, int k, int m0) {
                uint8_t *b = sB + (size_t)s * B_ST;
                if constexpr (F8) {
                    // the stage's planes {128 K, TM rows, planes} and scale words {TM rows, planes}
                    tma_load_3d(b, &tmX, k, m0, 0, &full[s]);
                    tma_load_2d(sW + (size_t)s * (F8_PLANES * TM), &tmS, m0, (k / (2 * BK)) * F8_PLANES, &full[s]);
                } else if (p.planes == 2) {
                    tma_load_3d(b, &tmX, k, m0, 0, &full[s]);
                } else {
                    tma_load_2d(b, &tmX, k, m0, &full[s]);
                }
            };
            // FP4: the exponent words of the tile's two 64-row halves (rows past the
            // matrix are not copied; the host keeps the row count a multiple of 4)
            int e_bytes0 = 0, e_bytes1 = 0;
            if (f4) {
                const int nt0 = tile0 % p.n_tiles, rows = p.swiglu_F ? 2 * p.swiglu_F : p.N;
                const int r0 = p.swiglu_F ? nt0 * 64 : nt0 * 128, r1 = p.swiglu_F ? p.swiglu_F + nt0 * 64 : nt0 * 128 + 64;
                e_bytes0 = 4 * max(0, min(64, rows - r0));
                e_bytes1 = 4 * max(0, min(64, rows - r1));
            }
            // bytes completing full[] (FP4 codes: the packed bytes the copy reads)
            const int a_tx = (f4 ? p.a_tx + e_bytes0 + e_bytes1 : A_ST) + B_ST + SW_ST;
            auto load_e = [&](int s, int kblk, int rowA0, int rowA1) {
                const uint32_t *src = p.w_bexp + (size_t)kblk * p.bs_rows + p.bs_row0;
                if (e_bytes0) bulk_load(sE + s * 128, src + rowA0, (uint32_t)e_bytes0, &full[s]);
                if (e_bytes1) bulk_load(sE + s * 128 + 64, src + rowA1, (uint32_t)e_bytes1, &full[s]);
            };
            int it = 0;     // global stage counter
            bool first = true, abort = false;
            for (int t = tile0; t < n_tiles_total && !abort; t += tstride) {
                const int nt = t % p.n_tiles, mt = t / p.n_tiles;
                const int rowA0 = g_wrow0 + (p.swiglu_F ? nt * 64 : nt * 128);
                const int rowA1 = g_wrow0 + (p.swiglu_F ? p.swiglu_F + nt * 64 : nt * 128 + 64);
                const int m0 = grouped ? g_row0 : mt * TM;
                int kk0 = 0;
                if (first) {
                    // weights do not depend on the previous kernel: start streaming them first
                    const int pre = min(nk, stages);
                    for (int i = 0; i < pre; ++i) {
                        uint8_t *a = sA + (size_t)i * A_ST;
                        mbar_expect_tx(&full[i], a_tx);
                        tma_load_2d_hint(a, &tmW, (kb + i) * kstep, rowA0, &full[i], wpol);
                        tma_load_2d_hint(a + A_ST / 2, &tmW, (kb + i) * kstep, rowA1, &full[i], wpol);
                        if (f4) load_e(i, kb + i, rowA0, rowA1);
                    }
                    if (!grouped) dep_wait(p.dep_ctr, p.dep_target, p.err);
                    for (int i = 0; i < pre; ++i) load_x(i, (kb + i) * kstep, m0);
                    kk0 = pre;
                    it = pre;
                    first = false;
                }
                for (int kk = kk0; kk < nk; ++kk, ++it) {
                    const int s = it % stages;
                    if (it >= stages && !mbar_wait(&empty[s], ((it / stages) & 1) ^ 1, p.err)) {
                        abort = true;
                        break;
                    }
                    const int k = (kb + kk) * kstep;
                    uint8_t *a = sA + (size_t)s * A_ST;
                    mbar_expect_tx(&full[s], a_tx);
                    tma_load_2d_hint(a, &tmW, k, rowA0, &full[s], wpol);
                    tma_load_2d_hint(a + A_ST / 2, &tmW, k, rowA1, &full[s], wpol);
                    if (f4) load_e(s, kb + kk, rowA0, rowA1);
                    load_x(s, k, m0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_bf16(wide ? 2 * TM : TM);
            int it = 0, lt = 0;  // global stage counter, local tile counter
            bool ok = true;
            for (int t = tile0; t < n_tiles_total && ok; t += tstride, ++lt) {
                const int b = lt & 1;
                if (lt >= 2 && !mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1, p.err)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t acc = tmem + (uint32_t)(b * NC1);
                for (int kk = 0; kk < nk; ++kk, ++it) {
                    const int s = it % stages;
                    if constexpr (F8) {
                        if (!mbar_wait(&full[s], (it / stages) & 1, p.err) ||
                            !mbar_wait(&sf_full[s], (it / stages) & 1, p.err)) {
                            ok = false;
                            break;
                        }
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        const uint64_t da = sw128_desc(smem_u32(sA + (size_t)s * A_ST));
                        const uint64_t db = sw128_desc(smem_u32(sB + (size_t)s * B_ST));
                        const uint32_t sfb = tmem_sfb + (uint32_t)(s * 4);
                        const uint32_t sfa = f4 ? tmem_sfa + (uint32_t)(s * 4) : tmem_sfa;
                        // A format: E4M3 (0) or, for FP4 weights, E2M1 (5), bits 7-9
                        const uint32_t afmt = f4 ? (5u << 7) : 0u;
#pragma unroll
                        for (int k32 = 0; k32 < 4; ++k32)  // 4 x K=32 over the stage's 128 K (+32 bytes each)
                            mma_mx(acc, da + (uint64_t)(k32 * 2), db + (uint64_t)(k32 * 2),
                                   idesc_mx(F8_PLANES * TM, k32) | afmt, sfa | ((uint32_t)k32 << 30),
                                   sfb | ((uint32_t)k32 << 30), (kk > 0 || k32 > 0) ? 1u : 0u);
                        mma_commit(&empty[s]);
                    } else {
                        if (!mbar_wait(&full[s], (it / stages) & 1, p.err)) {
                            ok = false;
                            break;
                        }
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        const uint64_t da = sw128_desc(smem_u32(sA + (size_t)s * A_BYTES));
                        const uint64_t db = sw128_desc(smem_u32(sB + (size_t)s * B_BYTES));
#pragma unroll
                        for (int k4 = 0; k4 < BK / 16; ++k4) {  // +32 bytes per K=16 step inside the swizzle row
                            mma_bf16(acc, da + (uint64_t)(k4 * 2), db + (uint64_t)(k4 * 2), idesc,
                                     (kk > 0 || k4 > 0) ? 1u : 0u);
                            if (p.planes == 2 && !wide)  // lo plane: TM rows (TM*128 bytes, a multiple of 1024) further on
                                mma_bf16(acc, da + (uint64_t)(k4 * 2), db + (uint64_t)((TM * 128) >> 4) + (uint64_t)(k4 * 2),
                                         idesc, 1u);
                        }
                        mma_commit(&empty[s]);
                    }
                }
                mma_commit(&acc_full[b]);
            }
        }
    } else {
        // ---------------- epilogue warps 2..5 ----------------
        const int q = warp & 3;
        const int n_local = q * 32 + lane;
        if constexpr (F8) copy_scales();
        if (p.dep_ctr) {
            if (threadIdx.x == 64) dep_wait(p.dep_ctr, p.dep_target, p.err);
            epi_bar();
        } else if (!grouped) {
            pdl_wait();
        }
        // F8: this thread's weight row and its scale
        float wsc = 1.f;
        if constexpr (F8) {
            const int nt0 = tile0 % p.n_tiles;
            const int row = p.swiglu_F ? (n_local < 64 ? nt0 * 64 + n_local : p.swiglu_F + nt0 * 64 + n_local - 64)
                                       : nt0 * 128 + n_local;
            const int rows = p.swiglu_F ? 2 * p.swiglu_F : p.N;
            wsc = row < rows ? p.w_scale[row] : 0.f;
        }
        // accumulator columns c..c+15 of a tile (F8: summed over the planes)
        auto load_acc = [&](uint32_t trow, int c, float *v) {
            if constexpr (F8) {
                tmem_ld16(trow + (uint32_t)c, v);
#pragma unroll
                for (int pl = 1; pl < F8_PLANES; ++pl) {
                    float t2[16];
                    tmem_ld16(trow + (uint32_t)(pl * TM + c), t2);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] += t2[j];
                }
            } else {
                acc_ld16(trow, c, lo_col, v);
            }
        };
        // K split: CTA `rank` of the cluster reduces and finishes columns [c_begin, c_end)
        const int rank = split ? (int)cluster_rank() : 0;
        const int cpr = split ? split_cols(TM, S) : TM;
        const int c_begin = split ? min(TM, rank * cpr) : 0;
        const int c_end = split ? min(TM, c_begin + cpr) : TM;
        int lt = 0, rs_mt = -1;
        for (int t = tile0; t < n_tiles_total; t += tstride, ++lt) {
            const int nt = t % p.n_tiles, mt = t / p.n_tiles;
            const int b = lt & 1;
            if (e.rs_ssq && mt != rs_mt) {  // before the accumulator is ready
                all_row_scales(e, mt * TM, TM, p.M, rsc);
                rs_mt = mt;
            }
            // inputs of this CTA's first epilogue chunk, while the mainloop streams
            if (c_end > c_begin) epi_prefetch<KIND, CH>(p, e, nt, n_local, mt * TM + c_begin, min(CH, c_end - c_begin), pre, smeta);
            const uint32_t trow = tmem + (uint32_t)(b * NC1) + ((uint32_t)(q * 32) << 16);
            const bool ok = mbar_wait(&acc_full[b], (lt >> 1) & 1, p.err) && nk > 0;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            float v[CH];
            if (!split) {
                for (int c = 0; c < TM; c += CH) {
                    if (ok) load_acc(trow, c, v);
                    else
#pragma unroll
                        for (int j = 0; j < CH; ++j) v[j] = 0.f;
                    if (F8)
#pragma unroll
                        for (int j = 0; j < CH; ++j) v[j] *= wsc;
                    if (c == TM - CH || TM == CH) {
                        // accumulator fully read: hand it back to the MMA warp
                        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc_empty[b]);
                    }
                    if (mt * TM + c < p.M || KIND != EPI_STORE)
                        epilogue_chunk<KIND>(p, e, nt, n_local, q, lane, mt * TM + c, CH, v, stg, red, smeta, rsc + c,
                                             c == 0 ? &pre : nullptr);
                }
            } else {
                // push this CTA's partial columns into the receive buffer of the CTA that
                // finishes them: recv[source rank][weight row][column - owner's c_begin],
                // four columns (one owner, cpr being a multiple of 4) per store
                cluster_wait();
                for (int c = 0; c < TM; c += CH) {
                    if (ok) load_acc(trow, c, v);
                    else
#pragma unroll
                        for (int j = 0; j < CH; ++j) v[j] = 0.f;
                    if (F8)
#pragma unroll
                        for (int j = 0; j < CH; ++j) v[j] *= wsc;
#pragma unroll
                    for (int g = 0; g < CH / 4; ++g) {
                        const int col = c + 4 * g, owner = col / cpr;
                        float *dst = recv + ((size_t)rank * 128 + n_local) * cpr + (col - owner * cpr);
                        st_cluster_v4(dst, (uint32_t)owner, v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                    }
                }
            }
        }
    }
    if (split) {
        // the pushes of every CTA are visible after the barrier (release / acquire);
        // afterwards no CTA touches another's shared memory, so one barrier suffices
        __syncwarp();
        if (warp < 2) cluster_wait();  // the epilogue warps waited before pushing
        cluster_sync_all();
        if (warp >= 2) {
            const int q = warp & 3;
            const int n_local = q * 32 + lane;
            const int nt = blockIdx.x, mt = blockIdx.y;
            const int rank = (int)cluster_rank();
            const int cpr = split_cols(TM, S);
            const int c_begin = min(TM, rank * cpr), c_end = min(TM, c_begin + cpr);
            // finish the owned columns with an epilogue no wider than needed
            auto finish = [&](auto width) {
                constexpr int W = decltype(width)::value;
                for (int c = c_begin; c < c_end; c += W) {
                    const int nc = min(W, c_end - c);
                    float v[CH];
#pragma unroll
                    for (int j = 0; j < CH; ++j) v[j] = 0.f;
                    for (int s2 = 0; s2 < S; ++s2) {  // in rank order: identical results run to run
                        const float *src = recv + ((size_t)s2 * 128 + n_local) * cpr + (c - c_begin);
#pragma unroll
                        for (int j = 0; j < W; ++j)
                            if (j < nc) v[j] += src[j];
                    }
                    epilogue_chunk<KIND, W>(p, e, nt, n_local, q, lane, mt * TM + c, nc, v, stg, red, smeta, rsc + c,
                                            c == c_begin ? &pre : nullptr);
                }
            };
            if (cpr <= 4) finish(std::integral_constant<int, 4>{});
            else if (cpr <= 8) finish(std::integral_constant<int, 8>{});
            else finish(std::integral_constant<int, CH>{});
        }
    }
    if (p.done_ctr) {  // every writer fences (generic and async proxy) before the signal
        __threadfence();
        fence_proxy_async_global();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (p.done_ctr && threadIdx.x == 0) {
        __threadfence();
        atomicAdd(p.done_ctr, 1);
    }
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

template <int TM, int KIND, bool F8, bool GR>
__global__ void __launch_bounds__(NT, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmS, const __grid_constant__ TcParams p,
                   const __grid_constant__ Epi<bf16> e, int stages) {
    if constexpr (GR) {
        // grouped (MoE experts): this CTA's expert, its rows and weight rows
        pdl_wait();  // the expert lists come from the bucketing kernel
        const int ex = p.g_touched[blockIdx.y];
        if (ex < 0) return;
        const int r0 = p.g_off[ex], m0 = (int)blockIdx.z * TM;
        const int nr = p.g_off[ex + 1] - r0;
        if (m0 >= nr) return;
        TcParams pg = p;
        Epi<bf16> eg = e;
        pg.M = min(TM, nr - m0);
        if (KIND == EPI_SWIGLU) eg.h += (size_t)(r0 + m0) * p.swiglu_F;
        if (KIND == EPI_STORE && p.g_list) eg.row_map = p.g_list + r0 + m0;
        gemm_tc_body<TM, KIND, F8, true>(tmW, tmX, tmS, pg, eg, stages, r0 + m0, ex * p.g_wrows);
    } else {
        gemm_tc_body<TM, KIND, F8, false>(tmW, tmX, tmS, p, e, stages, 0, 0);
    }
}

// MX planes of the activation rows of an FP8 projection: X [M][ld] bf16 (its
// low plane lo elements on when lo != 0), K columns.  Thread = 16 columns of a
// row (half a 32-column block; the other half in lane ^ 1).  Codes of plane p,
// row m, column k at codes[(p * mpad + m) * kpad + k]; the scale byte of
// (p, m, 32-column block b) is byte b % 4 of word ((b / 4) * F8_PLANES + p) *
// mpad + m of `words` (UE8M0: exponent + 127).
__global__ void __launch_bounds__(256) mx_quantize_kernel(const bf16 *__restrict__ X, int ld, size_t lo, int M, int K,
                                                          int mpad, int kpad, uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ words) {
    pdl_trigger();
    pdl_wait();  // X comes from the kernel before this one
    const int halves = K >> 4;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const bool in = u < (long long)M * halves;  // pairs of halves are both in or both out (halves is even)
    const int m = in ? (int)(u / halves) : 0, hb = in ? (int)(u % halves) : 0;
    const int k0 = hb * 16;
    float r[16];
    const bf16 *xr = X + (size_t)m * ld + k0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 hv = in ? *reinterpret_cast<const uint4 *>(xr + 8 * h) : make_uint4(0, 0, 0, 0);
        const uint4 lv = (in && lo) ? *reinterpret_cast<const uint4 *>(xr + lo + 8 * h) : make_uint4(0, 0, 0, 0);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&hw[i]));
            const float2 lf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&lw[i]));
            r[h * 8 + 2 * i] = hf.x + lf.x;
            r[h * 8 + 2 * i + 1] = hf.y + lf.y;
        }
    }
    uint4 code[F8_PLANES];
    int ex[F8_PLANES];
    mx_planes16<F8_PLANES>(r, code, ex);
    if (!in) return;
    const int blk = k0 >> 5;
#pragma unroll
    for (int pl = 0; pl < F8_PLANES; ++pl) {
        *reinterpret_cast<uint4 *>(codes + ((size_t)pl * mpad + m) * kpad + k0) = code[pl];
        if ((hb & 1) == 0) words[(((size_t)(blk >> 2) * F8_PLANES + pl) * mpad + m) * 4 + (blk & 3)] = (uint8_t)(ex[pl] + 127);
    }
}

// final argmax over the per-tile partials of each row
__global__ void lm_argmax_kernel(const float2 *__restrict__ part, int n_tiles, int R, int mode, int B, int *idx,
                                 DevStats *stats) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    if (mode == 1 && (r % B) == 0) return;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
        const float2 v = part[(size_t)t * R + r];
        argmax_merge(bv, bi, v.x, __float_as_int(v.y));
    }
    __shared__ float sv[32];
    __shared__ int si[32];
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        argmax_merge(bv, bi, v2, i2);
    }
    if ((threadIdx.x & 31) == 0) {
        sv[threadIdx.x >> 5] = bv;
        si[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bv = sv[0];
        bi = si[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) argmax_merge(bv, bi, sv[w], si[w]);
        if (!isfinite(bv) && stats) atomicOr(&stats->status, 1);
        if (bi == 0x7fffffff) bi = 0;
        if (mode == 0) idx[r] = bi;
        else idx[(r / B) * (B - 1) + (r % B) - 1] = bi;
    }
}

}  // namespace tc

void launch_lm_argmax(const float2 *part, int n_tiles, int R, int mode, int B, int *idx, DevStats *stats,
                      cudaStream_t s) {
    if (R <= 0) return;
    launch_k(tc::lm_argmax_kernel, dim3(R), dim3(256), 0, s, 1, part, n_tiles, R, mode, B, idx, stats);
}

int gemm_tc_workspace_floats(int max_rows, int max_n) {
    (void)max_rows;
    (void)max_n;
    return 8 << 20;  // 32 MB of split-K partials
}

int gemm_tc_semaphores() { return 1 << 16; }

bool &pdl_enabled() {
    // DFLASH_PDL=0 launches every kernel without programmatic dependent launch
    static bool on = [] {
        const char *v = getenv("DFLASH_PDL");
        return !(v && v[0] == '0');
    }();
    return on;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

template <>
bool GemmTC<bf16>::supports(int M, int N, int K) const {
    return M >= 1 && N >= 1 && K >= 8 && (K % 8) == 0;
}
template <>
bool GemmTC<float>::supports(int, int, int) const {
    return false;
}

template <typename T>
int GemmTC<T>::init(float *w, int wf, int *sm, int ns) {
    ws = w;
    ws_floats = wf;
    sem = sm;
    n_sem = ns;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (std::is_same<T, bf16>::value && !get_encode()) {
        err = "cuTensorMapEncodeTiled entry point unavailable";
        return 1;
    }
    return 0;
}

template <typename T>
const CUtensorMap *GemmTC<T>::tensor_map(const void *ptr, int rows, int cols, int ld, int box_rows,
                                         size_t plane_stride, bool fp8) {
    char key[128];
    snprintf(key, sizeof key, "%p/%d/%d/%d/%d/%zu/%d", ptr, rows, cols, ld, box_rows, plane_stride, fp8 ? 1 : 0);
    auto it = maps.find(key);
    if (it != maps.end()) return &it->second;
    if (maps.size() > 4096) maps.clear();
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    const cuuint32_t rank = plane_stride ? 3 : 2;
    const size_t es = fp8 ? 1 : sizeof(bf16);
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, 2};
    cuuint64_t strides[2] = {(cuuint64_t)ld * es, (cuuint64_t)plane_stride * es};
    // one 128-byte swizzle row per box row: 64 bf16 or 128 FP8 codes
    cuuint32_t box[3] = {(cuuint32_t)(fp8 ? 2 * tc::BK : tc::BK), (cuuint32_t)box_rows, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    if (plane_stride && (plane_stride * sizeof(bf16)) % 16) {
        err = "lo-plane offset is not a multiple of 16 bytes";
        return nullptr;
    }
    CUresult r = get_encode()(&m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                              const_cast<void *>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed";
        return nullptr;
    }
    return &(maps[key] = m);
}

template <typename T>
const CUtensorMap *GemmTC<T>::fp4_map(const void *ptr, int rows, int cols, int box_rows) {
    char key[96];
    snprintf(key, sizeof key, "fp4/%p/%d/%d/%d", ptr, rows, cols, box_rows);
    auto it = maps.find(key);
    if (it != maps.end()) return &it->second;
    if (maps.size() > 4096) maps.clear();
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    // dims count 4-bit elements; the row stride is in bytes (cols / 2)
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols / 2};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = get_encode()(&m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void *>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed (FP4 weights)";
        return nullptr;
    }
    return &(maps[key] = m);
}

// Tensor map of the MX activation planes of an M x K projection input:
// (K bytes, M rows, planes), box {128 K, tm rows, planes}, 128-byte swizzle.
// Rows >= M and columns >= K read as zero codes.
template <typename T>
const CUtensorMap *GemmTC<T>::mx_map_codes(int M, int K, int tm) {
    char key[96];
    snprintf(key, sizeof key, "mxc/%p/%d/%d/%d", (void *)mx_codes, M, K, tm);
    auto it = maps.find(key);
    if (it != maps.end()) return &it->second;
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)M, (cuuint64_t)tc::F8_PLANES};
    cuuint64_t strides[2] = {(cuuint64_t)mx_kpad, (cuuint64_t)mx_kpad * mx_mpad};
    cuuint32_t box[3] = {128, (cuuint32_t)tm, (cuuint32_t)tc::F8_PLANES};
    cuuint32_t estr[3] = {1, 1, 1};
    if (get_encode()(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, mx_codes, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed (MX planes)";
        return nullptr;
    }
    return &(maps[key] = m);
}

// Tensor map of the MX scale words: (M words, stages x planes rows), box
// {tm words, planes}: a stage's words land as [plane][row].
template <typename T>
const CUtensorMap *GemmTC<T>::mx_map_words(int M, int K, int tm) {
    char key[96];
    snprintf(key, sizeof key, "mxw/%p/%d/%d/%d", (void *)mx_words, M, K, tm);
    auto it = maps.find(key);
    if (it != maps.end()) return &it->second;
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    const int ks = (K + 127) / 128;
    cuuint64_t dims[2] = {(cuuint64_t)M, (cuuint64_t)ks * tc::F8_PLANES};
    cuuint64_t strides[1] = {(cuuint64_t)mx_mpad * 4};
    cuuint32_t box[2] = {(cuuint32_t)tm, (cuuint32_t)tc::F8_PLANES};
    cuuint32_t estr[2] = {1, 1};
    if (get_encode()(&m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, mx_words, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed (MX scales)";
        return nullptr;
    }
    return &(maps[key] = m);
}

template <int TM, int KIND, bool F8>
static void launch_tm(const CUtensorMap *mw, const CUtensorMap *mx, const CUtensorMap *ms, const TcParams &p,
                      const Epi<bf16> &e, int stages, size_t smem, cudaStream_t s, int grid_x) {
    auto kern = tc::gemm_tc_kernel<TM, KIND, F8, false>;
    ensure_smem_attr((const void *)kern);
    (void)grid_x;
    dim3 grid(p.n_tiles, p.m_tiles, p.splits);
    launch_k(kern, grid, dim3(tc::NT), smem, s, p.splits, *mw, *mx, *ms, p, e, stages);
}

template <int TM, bool F8>
static void launch_kind(int kind, const CUtensorMap *mw, const CUtensorMap *mx, const CUtensorMap *ms, const TcParams &p,
                        const Epi<bf16> &e, int stages, size_t smem, cudaStream_t s, int gx) {
    switch (kind) {
        case EPI_STORE: launch_tm<TM, EPI_STORE, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
        case EPI_QKV: launch_tm<TM, EPI_QKV, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
        case EPI_RESID: launch_tm<TM, EPI_RESID, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
        case EPI_SWIGLU: launch_tm<TM, EPI_SWIGLU, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
        case EPI_NORMOUT: launch_tm<TM, EPI_NORMOUT, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
        default: launch_tm<TM, EPI_LOGITS, F8>(mw, mx, ms, p, e, stages, smem, s, gx); break;
    }
}

template <typename T>
TcPlan GemmTC<T>::plan(int M, int N, int K, int kind, int F, bool f8, int planes, bool f4) const {
    const bool swiglu = kind == EPI_SWIGLU;
    TcPlan pl;
    int TM = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    if (tune_tm_max >= 16) {
        TM = std::min(TM, tune_tm_max);
    } else if (TM > 64) {
        // many activation rows (batched decode, prefill chunks): the largest row tile
        // up to 128 that still gives every SM a tile; the weight tile is then re-read
        // per row tile, from L2 (measured: one CTA per weight tile left most SMs
        // idle).  128 rows at most: a 256-row tile's two-stage ring (~176 KB) holds
        // one CTA per SM, while two ~110 KB CTAs of 128 rows stream better
        // (measured on B200, Qwen3-8B shape: batch 8 12.3 -> 10.6 ms per step,
        // batch 32 gate/up 245 -> 217 us and LM head 1648 -> 1409 us)
        TM = std::min(TM, 128);
        const int nt = swiglu ? (F + 63) / 64 : (N + 127) / 128;
        while (TM > 64 && nt * ((M + TM - 1) / TM) < num_sms) TM /= 2;
    }
    // FP8: N = 4 planes x TM <= 128 keeps the accumulator and the scale columns in
    // 256 TMEM columns (two CTAs per SM); larger M takes several row tiles
    if (f8) TM = std::min(TM, 32);
    pl.TM = TM;
    pl.n_tiles = swiglu ? (F + 63) / 64 : (N + 127) / 128;
    pl.m_tiles = (M + TM - 1) / TM;
    pl.kstep = f8 ? 2 * tc::BK : tc::BK;  // K per stage: 128 FP8 codes or 64 bf16 values per weight row
    pl.k_steps = (K + pl.kstep - 1) / pl.kstep;
    const int tiles = pl.n_tiles * pl.m_tiles;
    // a stage: the weight tile + the activation tile(s) (FP8: codes + activation planes + scale words)
    // (FP4: the same 16 KB of weight codes in shared memory, plus the 128 rows' exponent words)
    const int stage_bytes = f8 ? tc::F8_A_BYTES + tc::F8_PLANES * TM * (128 + 4) + (f4 ? 512 : 0)
                               : tc::A_BYTES + TM * 128 * planes;
    // fixed area: alignment, epilogue staging, barriers
    const int fixed = 1024 + 128 * tc::STG_LD * 4 + 4 * tc::CH * 8 + tc::CH * 16 + tc::RS_MAX * 4 + 64 * 8 + 64 + 16 * 8;
    // Measured on B200 (decode shapes, M = 16, whole decode iteration): every
    // projection streams best with ~110 KB CTAs, two of which fit on an SM;
    // projections with fewer tiles than that split K over a cluster (up to 8
    // CTAs) to fill both slots of every SM.  Larger (150 KB, one CTA per SM)
    // rings were faster for a projection timed alone but 0.5 ms per iteration
    // slower in the pipeline; filling one slot per SM was 0.2 ms slower.
    int splits = 1;
    // the K split aims to fill two ~110 KB CTAs per SM (measured best in the decode
    // pipeline), as far as clusters allow: a cluster is placed whole inside one GPC,
    // and on B200 one wave of these CTAs held 43 clusters of 6 or 32 clusters of 8
    // (about 256 CTAs, not the 296 slots on paper); 48 clusters of 6 ran as 43 + 5
    const int slots = tune_ctas_per_sm > 0 ? num_sms * tune_ctas_per_sm : std::min(2 * num_sms, 256);
    if (kind != EPI_LOGITS && tiles < slots && pl.k_steps >= 4) {
        splits = std::max(1, std::min({8, pl.k_steps / 2, slots / std::max(1, tiles)}));
        if (tune_splits > 0) splits = std::min(8, tune_splits);
        const int k_per = (pl.k_steps + splits - 1) / splits;
        splits = (pl.k_steps + k_per - 1) / k_per;
    }
    if (TM > 64) splits = 1;  // keeps the split-K receive buffer (S x 128 x TM/S floats) small
    pl.splits = splits;
    // split-K receive buffer [S][128][ceil(TM/S)] floats, placed after the fixed area
    const int recv_bytes = splits > 1 ? splits * 128 * tc::split_cols(TM, splits) * 4 + 64 : 0;
    // two CTAs per SM up to 128-row tiles (128 rows: a two-stage ring of 48 KB stages)
    int budget = splits > 1 ? 110 * 1024 : (TM <= 128 ? 112 * 1024 : 200 * 1024);
    if (splits > 1 && tune_split_smem_kb > 0) budget = tune_split_smem_kb * 1024;
    if (splits == 1 && tune_smem_kb > 0) budget = tune_smem_kb * 1024;
    pl.stages = std::max(2, std::min(16, (budget - fixed - recv_bytes) / stage_bytes));
    pl.smem = (size_t)fixed + (size_t)recv_bytes + (size_t)pl.stages * stage_bytes;
    return pl;
}

template <>
int GemmTC<bf16>::run(const bf16 *X, int ldx, int M, const void *W, int N, int K, const Epi<bf16> &e,
                      cudaStream_t s, const int *dep_ctr, int dep_target, int *done_ctr, const float *w_scale,
                      const uint8_t *w_bexp, int bs_rows, int bs_row0) {
    const bool swiglu = e.kind == EPI_SWIGLU;
    const bool f8 = w_scale != nullptr;
    const TcPlan pl = plan(M, N, K, e.kind, e.F, f8, e.lo ? 2 : 1, f8 && w_bexp != nullptr);
    const int TM = pl.TM, splits = pl.splits, stages = pl.stages;
    const size_t smem = pl.smem;
    TcParams p;
    memset(&p, 0, sizeof p);
    p.M = M;
    p.N = N;
    p.K = K;
    p.swiglu_F = swiglu ? e.F : 0;
    p.n_tiles = pl.n_tiles;
    p.m_tiles = pl.m_tiles;
    p.k_steps = pl.k_steps;
    p.planes = e.lo ? 2 : 1;
    p.w_scale = w_scale;
    const bool f4 = f8 && w_bexp != nullptr;
    if (f4) {
        p.w_bexp = reinterpret_cast<const uint32_t *>(w_bexp);
        p.bs_rows = bs_rows;
        p.bs_row0 = bs_row0;
        // a stage's codes complete the barrier with the bytes the copy reads (8 KB
        // packed), not the 16 KB they fill in shared memory (measured on B200: with
        // 16 KB the barrier never completed)
        p.a_tx = tc::F8_A_BYTES / 2;
    }
    p.splits = splits;
    p.err = err_word;
    p.lm_part = lm_part;
    p.keep_logits = keep_logits;
    p.dep_ctr = dep_ctr;
    p.dep_target = dep_target;
    p.done_ctr = done_ctr;
    const int grid_x = p.n_tiles;  // one tile per CTA
    if (f4 && (K % 128 || ((swiglu ? 2 * e.F : N) % 4) || bs_rows % 4 || bs_row0 % 4 ||
               (reinterpret_cast<uintptr_t>(W) & 31) || (reinterpret_cast<uintptr_t>(w_bexp) & 15))) {
        failed = true;
        err = "FP4 projection: K must be a multiple of 128, the row counts of 4, the codes 32-byte aligned";
        return 0;
    }
    const CUtensorMap *mw = f4 ? fp4_map(W, swiglu ? 2 * e.F : N, K, 64) : tensor_map(W, swiglu ? 2 * e.F : N, K, K, 64, 0, f8);
    const CUtensorMap *mx = nullptr, *ms = nullptr;
    if (f8) {
        // the activation rows as MX planes (a kernel of their own, before the projection)
        if (!mx_codes || M > mx_mpad || K > mx_kpad || K % 32 || ldx % 8) {
            failed = true;
            err = "FP8 projection: activation rows do not fit the MX buffers";
            return 0;
        }
        const int threads = M * (K / 16);
        launch_k(tc::mx_quantize_kernel, dim3((threads + 255) / 256), dim3(256), 0, s, 1, X, ldx, e.lo, M, K,
                 mx_mpad, mx_kpad, mx_codes, mx_words);
        mx = mx_map_codes(M, K, TM);
        ms = mx_map_words(M, K, TM);
    } else {
        mx = tensor_map(X, M, K, ldx, TM, e.lo);
        ms = mx;
    }
    if (!mw || !mx || !ms) {
        failed = true;
        return 0;
    }
    if (f8) {
        switch (TM) {
            case 16: launch_kind<16, true>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
            default: launch_kind<32, true>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
        }
    } else {
        switch (TM) {
            case 16: launch_kind<16, false>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
            case 32: launch_kind<32, false>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
            case 64: launch_kind<64, false>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
            case 128: launch_kind<128, false>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
            default: launch_kind<256, false>(e.kind, mw, mx, ms, p, e, stages, smem, s, grid_x); break;
        }
    }
    return p.n_tiles * p.m_tiles * p.splits;
}

template <>
int GemmTC<float>::run(const float *, int, int, const void *, int, int, const Epi<float> &, cudaStream_t,
                       const int *, int, int *, const float *, const uint8_t *, int, int) {
    return 0;
}

template <>
int GemmTC<bf16>::run_grouped(const bf16 *X, int ldx, int n_pairs, const bf16 *W, int wrows, int N, int K,
                              const Epi<bf16> &e, const int *off, const int *touched, const int *list, int E,
                              int max_rows, cudaStream_t s) {
    const bool swiglu = e.kind == EPI_SWIGLU;
    const int TM = max_rows <= 16 ? 16 : max_rows <= 32 ? 32 : 64;
    TcParams p;
    memset(&p, 0, sizeof p);
    p.M = n_pairs;
    p.N = N;
    p.K = K;
    p.swiglu_F = swiglu ? e.F : 0;
    p.n_tiles = swiglu ? (e.F + 63) / 64 : (N + 127) / 128;
    p.m_tiles = (max_rows + TM - 1) / TM;
    p.k_steps = (K + tc::BK - 1) / tc::BK;
    p.planes = e.lo ? 2 : 1;
    p.splits = 1;
    p.err = err_word;
    p.g_off = off;
    p.g_touched = touched;
    p.g_list = list;
    p.g_wrows = wrows;
    const int stage_bytes = tc::A_BYTES + TM * 128 * p.planes;
    const int fixed = 1024 + 128 * tc::STG_LD * 4 + 4 * tc::CH * 8 + tc::CH * 16 + tc::RS_MAX * 4 + 64 * 8 + 64 + 16 * 8;
    const int stages = std::max(2, std::min(16, (112 * 1024 - fixed) / stage_bytes));
    const size_t smem = (size_t)fixed + (size_t)stages * stage_bytes;
    const CUtensorMap *mw = tensor_map(W, E * wrows, K, K, 64);
    const CUtensorMap *mx = tensor_map(X, n_pairs, K, ldx, TM, e.lo);
    if (!mw || !mx) {
        failed = true;
        return 0;
    }
    auto go = [&](auto tm_c) {
        constexpr int T_ = decltype(tm_c)::value;
        auto kern = swiglu ? tc::gemm_tc_kernel<T_, EPI_SWIGLU, false, true> : tc::gemm_tc_kernel<T_, EPI_STORE, false, true>;
        ensure_smem_attr((const void *)kern);
        launch_k(kern, dim3(p.n_tiles, E, p.m_tiles), dim3(tc::NT), smem, s, 1, *mw, *mx, *mx, p, e, stages);
    };
    if (TM == 16) go(std::integral_constant<int, 16>{});
    else if (TM == 32) go(std::integral_constant<int, 32>{});
    else go(std::integral_constant<int, 64>{});
    return p.n_tiles * E * p.m_tiles;
}

template <>
int GemmTC<float>::run_grouped(const float *, int, int, const float *, int, int, int, const Epi<float> &, const int *,
                               const int *, const int *, int, int, cudaStream_t) {
    return 0;
}

template struct GemmTC<bf16>;
template struct GemmTC<float>;

template <>
bool moe_tc_supported<bf16>() {
    return false;
}
template <>
bool moe_tc_supported<float>() {
    return false;
}

template <typename T>
void run_moe_tc(const T *, int, int, int, const int *, const T *, const T *, int, int, int, T *, float *, GemmTC<T> &,
                cudaStream_t) {}
template void run_moe_tc<bf16>(const bf16 *, int, int, int, const int *, const bf16 *, const bf16 *, int, int, int,
                               bf16 *, float *, GemmTC<bf16> &, cudaStream_t);
template void run_moe_tc<float>(const float *, int, int, int, const int *, const float *, const float *, int, int, int,
                                float *, float *, GemmTC<float> &, cudaStream_t);

}  // namespace dfl
