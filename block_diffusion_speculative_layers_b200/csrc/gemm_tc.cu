// gemm_tc.cu -- tensor-core weight-streaming projection for bf16 models on
// sm_100a: TMA (SWIZZLE_128B) -> shared-memory ring -> tcgen05.mma (accumulator
// in TMEM) -> fused epilogue.
//
// Roles per CTA (192 threads):
//   warp 0      one thread issues TMA loads of the weight tile (two 64-row
//               boxes) and the activation tile into a ring of stages;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=TM,
//               K=16) and commits each consumed stage back to the producer;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = weight rows), split-K reduction when the
//               K range is split, then the fused epilogue (store / RoPE + KV
//               write / residual + taps / SwiGLU / per-tile argmax).
// Split-K partials are summed by the last-arriving CTA of a tile in split
// order, so results are identical run to run.  Every mbarrier wait is bounded
// (2 s of %globaltimer); on expiry the CTA records an error bit and drains.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>

#include "gemm_tc.h"

namespace dfl {
namespace tc {

constexpr int BK = 64;                 // bf16 K elements per stage = one 128-byte swizzle row
constexpr int A_BYTES = 128 * BK * 2;  // 16 KB weight tile per stage
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

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// ---------------------------------------------------------------------------
// fused epilogue on one chunk of CH accumulator columns (activation rows
// m0c .. m0c+CH-1) for weight row n_local of the tile
// ---------------------------------------------------------------------------
template <int KIND>
__device__ __forceinline__ void epilogue_chunk(const TcParams &p, const Epi<bf16> &e, int nt, int n_local, int q,
                                               int lane, int m0c, const float *v, float *stg, float2 *red) {
    const int M = p.M;
    if (KIND == EPI_STORE || KIND == EPI_RESID) {
        const int n = nt * 128 + n_local;
        if (n < p.N) {
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                const int m = m0c + j;
                if (m >= M) break;
                if (KIND == EPI_STORE) {
                    e.Y[(size_t)m * e.ldy + n] = v[j];
                } else {
                    float *xp = e.x + (size_t)m * p.N + n;
                    const float nx = *xp + v[j];
                    *xp = nx;
                    if (e.taps.n) {
                        const int trow = e.meta[m].aux;
                        for (int t = 0; t < e.taps.n; ++t)
                            e.taps.base[(size_t)trow * e.taps.ld + e.taps.col[t] + n] = __float2bfloat16_rn(nx);
                    }
                }
            }
        }
    } else if (KIND == EPI_LOGITS) {
        const int n = nt * 128 + n_local;
        const bool ok = n < p.N;
#pragma unroll
        for (int j = 0; j < CH; ++j) {
            const int m = m0c + j;
            if (p.keep_logits && ok && m < M) e.Y[(size_t)m * e.ldy + n] = v[j];
            float bv = ok ? v[j] : -INFINITY;
            int bi = ok ? n : 0x7fffffff;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
                const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
                argmax_merge(bv, bi, v2, i2);
            }
            if (lane == 0) red[q * CH + j] = make_float2(bv, __int_as_float(bi));
        }
        epi_bar();
        if (threadIdx.x >= 64 && threadIdx.x < 64 + CH) {
            const int j = threadIdx.x - 64;
            const int m = m0c + j;
            float bv = red[j].x;
            int bi = __float_as_int(red[j].y);
            for (int qq = 1; qq < 4; ++qq) argmax_merge(bv, bi, red[qq * CH + j].x, __float_as_int(red[qq * CH + j].y));
            if (m < M) p.lm_part[(size_t)nt * p.M + m] = make_float2(bv, __int_as_float(bi));
        }
        epi_bar();
    } else if (KIND == EPI_SWIGLU) {
#pragma unroll
        for (int j = 0; j < CH; ++j) stg[n_local * STG_LD + j] = v[j];
        epi_bar();
        if (n_local < 64) {
            const int f = nt * 64 + n_local;
            if (f < p.swiglu_F) {
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    const int m = m0c + j;
                    if (m >= M) break;
                    // gate and up are bf16-rounded like any projection output feeding a GEMM
                    const float up = stg[(n_local + 64) * STG_LD + j];
                    e.h[(size_t)m * p.swiglu_F + f] = __float2bfloat16_rn(silu_f(v[j]) * up);
                }
            }
        }
        epi_bar();
    } else if (KIND == EPI_QKV) {
#pragma unroll
        for (int j = 0; j < CH; ++j) stg[n_local * STG_LD + j] = v[j];
        epi_bar();
        const int hd = e.hd, half = hd >> 1;
        const int qd = e.nq * hd, kd = e.nkv * hd;
        const int cg = e.col0 + nt * 128 + n_local;  // row of [Wq; Wk; Wv]
        const int nloc_ok = (nt * 128 + n_local) < p.N;
        if (nloc_ok) {
            const int head_base = (cg / hd) * hd;
            const int d = cg - head_base;
            const int partner = n_local + (d < half ? half : -half);
            const int i = d < half ? d : d - half;
            const bool is_q = cg < qd, is_k = !is_q && cg < qd + kd;
#pragma unroll 4
            for (int j = 0; j < CH; ++j) {
                const int m = m0c + j;
                if (m >= M) break;
                const bool ctx = m >= e.R_blk;
                const RowMeta mt = ctx ? e.ctx_meta[m - e.R_blk] : e.meta[m];
                if (ctx && (is_q || !mt.aux)) continue;
                float out = v[j];
                if (is_q || is_k) {
                    const float2 cs = e.rope[(size_t)mt.pos * half + i];
                    const float other = stg[partner * STG_LD + j];
                    out = d < half ? v[j] * cs.x - other * cs.y : v[j] * cs.x + other * cs.y;
                }
                if (is_q) {
                    e.q_out[(size_t)m * qd + cg] = __float2bfloat16_rn(out);
                } else {
                    const int hh = is_k ? (cg - qd) / hd : (cg - qd - kd) / hd;
                    bf16 *dst = (is_k ? e.kc : e.vc) + (((size_t)mt.seq * e.nkv + hh) * e.max_len + mt.pos) * hd;
                    dst[d] = __float2bfloat16_rn(out);
                }
            }
        }
        epi_bar();
    }
}

template <int TM, int KIND>
__global__ void __launch_bounds__(NT, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, TcParams p,
                   Epi<bf16> e, int stages) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int B_BYTES = TM * 128;
    constexpr int NCOLS = TM < 32 ? 32 : TM;
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)stages * A_BYTES;
    float *stg = (float *)(sB + (size_t)stages * B_BYTES);
    float2 *red = (float2 *)(stg + 128 * STG_LD);
    uint64_t *full = (uint64_t *)(red + 4 * CH);
    uint64_t *empty = full + stages;
    uint64_t *done = empty + stages;
    uint32_t *tmem_slot = (uint32_t *)(done + 1);
    int *flag = (int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = blockIdx.x, mt = blockIdx.y, sp = blockIdx.z;
    const int k_per = (p.k_steps + p.splits - 1) / p.splits;
    const int kb = sp * k_per, ke = min(p.k_steps, kb + k_per);
    const int nk = ke - kb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        flag[0] = 0;
        flag[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(NCOLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            const int rowA0 = p.swiglu_F ? nt * 64 : nt * 128;
            const int rowA1 = p.swiglu_F ? p.swiglu_F + nt * 64 : nt * 128 + 64;
            const int m0 = mt * TM;
            for (int it = 0; it < nk; ++it) {
                const int s = it % stages;
                if (it >= stages && !mbar_wait(&empty[s], ((it / stages) & 1) ^ 1, p.err)) {
                    flag[1] = 1;
                    break;
                }
                if (flag[1]) break;
                const int k = (kb + it) * BK;
                uint8_t *a = sA + (size_t)s * A_BYTES;
                mbar_expect_tx(&full[s], A_BYTES + B_BYTES);
                tma_load_2d(a, &tmW, k, rowA0, &full[s]);
                tma_load_2d(a + A_BYTES / 2, &tmW, k, rowA1, &full[s]);
                tma_load_2d(sB + (size_t)s * B_BYTES, &tmX, k, m0, &full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_bf16(TM);
            for (int it = 0; it < nk; ++it) {
                const int s = it % stages;
                if (!mbar_wait(&full[s], (it / stages) & 1, p.err)) {
                    flag[1] = 1;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint64_t da = sw128_desc(smem_u32(sA + (size_t)s * A_BYTES));
                const uint64_t db = sw128_desc(smem_u32(sB + (size_t)s * B_BYTES));
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes per K=16 step inside the swizzle row
                    mma_bf16(tmem, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            mma_commit(done);
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;
        const int n_local = q * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        const bool ok = mbar_wait(done, 0, p.err);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int tile = mt * p.n_tiles + nt;
        float v[CH];
        bool last = true;
        if (p.splits > 1) {
            float *mine = p.ws + ((size_t)tile * p.splits + sp) * (size_t)TM * 128;
            for (int c = 0; c < TM; c += CH) {
                if (ok) tmem_ld16(trow + c, v);
                else
                    for (int j = 0; j < CH; ++j) v[j] = 0.f;
#pragma unroll
                for (int j = 0; j < CH; ++j) mine[(size_t)(c + j) * 128 + n_local] = v[j];
            }
            __threadfence();
            epi_bar();
            if (threadIdx.x == 64) {
                const int old = atomicAdd(&p.sem[tile], 1);
                flag[0] = (old == p.splits - 1) ? 1 : 0;
            }
            epi_bar();
            last = flag[0] != 0;
            if (last) __threadfence();
        }
        if (last) {
            for (int c = 0; c < TM; c += CH) {
                if (p.splits > 1) {
#pragma unroll
                    for (int j = 0; j < CH; ++j) v[j] = 0.f;
                    for (int s2 = 0; s2 < p.splits; ++s2) {
                        const float *src = p.ws + ((size_t)tile * p.splits + s2) * (size_t)TM * 128;
#pragma unroll
                        for (int j = 0; j < CH; ++j) v[j] += __ldcg(src + (size_t)(c + j) * 128 + n_local);
                    }
                } else if (ok) {
                    tmem_ld16(trow + c, v);
                } else {
                    for (int j = 0; j < CH; ++j) v[j] = 0.f;
                }
                const int m0c = mt * TM + c;
                if (m0c < p.M || KIND == EPI_LOGITS || KIND == EPI_SWIGLU || KIND == EPI_QKV)
                    epilogue_chunk<KIND>(p, e, nt, n_local, q, lane, m0c, v, stg, red);
            }
            if (p.splits > 1 && threadIdx.x == 64) p.sem[tile] = 0;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS));
    }
}

// final argmax over the per-tile partials of each row
__global__ void lm_argmax_kernel(const float2 *__restrict__ part, int n_tiles, int R, int mode, int B, int *idx,
                                 DevStats *stats) {
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
    tc::lm_argmax_kernel<<<R, 256, 0, s>>>(part, n_tiles, R, mode, B, idx, stats);
}

int gemm_tc_workspace_floats(int max_rows, int max_n) {
    (void)max_rows;
    (void)max_n;
    return 8 << 20;  // 32 MB of split-K partials
}

int gemm_tc_semaphores() { return 1 << 16; }

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
const CUtensorMap *GemmTC<T>::tensor_map(const void *ptr, int rows, int cols, int ld, int box_rows) {
    char key[96];
    snprintf(key, sizeof key, "%p/%d/%d/%d/%d", ptr, rows, cols, ld, box_rows);
    auto it = maps.find(key);
    if (it != maps.end()) return &it->second;
    if (maps.size() > 4096) maps.clear();
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * sizeof(bf16)};
    cuuint32_t box[2] = {(cuuint32_t)tc::BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = get_encode()(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed";
        return nullptr;
    }
    return &(maps[key] = m);
}

template <int TM, int KIND>
static void launch_tm(const CUtensorMap *mw, const CUtensorMap *mx, const TcParams &p, const Epi<bf16> &e,
                      int stages, size_t smem, cudaStream_t s) {
    auto kern = tc::gemm_tc_kernel<TM, KIND>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        attr_set = true;
    }
    dim3 grid(p.n_tiles, p.m_tiles, p.splits);
    kern<<<grid, tc::NT, smem, s>>>(*mw, *mx, p, e, stages);
}

template <int TM>
static void launch_kind(int kind, const CUtensorMap *mw, const CUtensorMap *mx, const TcParams &p,
                        const Epi<bf16> &e, int stages, size_t smem, cudaStream_t s) {
    switch (kind) {
        case EPI_STORE: launch_tm<TM, EPI_STORE>(mw, mx, p, e, stages, smem, s); break;
        case EPI_QKV: launch_tm<TM, EPI_QKV>(mw, mx, p, e, stages, smem, s); break;
        case EPI_RESID: launch_tm<TM, EPI_RESID>(mw, mx, p, e, stages, smem, s); break;
        case EPI_SWIGLU: launch_tm<TM, EPI_SWIGLU>(mw, mx, p, e, stages, smem, s); break;
        default: launch_tm<TM, EPI_LOGITS>(mw, mx, p, e, stages, smem, s); break;
    }
}

template <>
void GemmTC<bf16>::run(const bf16 *X, int ldx, int M, const bf16 *W, int N, int K, const Epi<bf16> &e,
                       cudaStream_t s) {
    const bool swiglu = e.kind == EPI_SWIGLU;
    int TM = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    TcParams p;
    memset(&p, 0, sizeof p);
    p.M = M;
    p.N = N;
    p.K = K;
    p.swiglu_F = swiglu ? e.F : 0;
    p.n_tiles = swiglu ? (e.F + 63) / 64 : (N + 127) / 128;
    p.m_tiles = (M + TM - 1) / TM;
    p.k_steps = (K + tc::BK - 1) / tc::BK;
    const int tiles = p.n_tiles * p.m_tiles;
    int splits = 1;
    if (e.kind != EPI_LOGITS) {
        const int target = 2 * num_sms;
        splits = std::max(1, std::min(p.k_steps / 4, target / std::max(1, tiles)));
        while (splits > 1 && ((size_t)tiles * splits * TM * 128 > (size_t)ws_floats || tiles > n_sem)) --splits;
        const int k_per = (p.k_steps + splits - 1) / splits;
        splits = (p.k_steps + k_per - 1) / k_per;
    }
    p.splits = splits;
    p.ws = ws;
    p.sem = sem;
    p.err = err_word;
    p.lm_part = lm_part;
    p.keep_logits = keep_logits;
    const CUtensorMap *mw = tensor_map(W, swiglu ? 2 * e.F : N, K, K, 64);
    const CUtensorMap *mx = tensor_map(X, M, K, ldx, TM);
    if (!mw || !mx) return;
    const int stage_bytes = tc::A_BYTES + TM * 128;
    const int fixed = 1024 + 128 * tc::STG_LD * 4 + 4 * tc::CH * 8 + 64 * 8 + 64;
    const int budget = TM <= 64 ? 112 * 1024 : 200 * 1024;
    const int stages = std::max(2, std::min(8, (budget - fixed) / stage_bytes));
    const size_t smem = (size_t)fixed + (size_t)stages * stage_bytes;
    switch (TM) {
        case 16: launch_kind<16>(e.kind, mw, mx, p, e, stages, smem, s); break;
        case 32: launch_kind<32>(e.kind, mw, mx, p, e, stages, smem, s); break;
        case 64: launch_kind<64>(e.kind, mw, mx, p, e, stages, smem, s); break;
        case 128: launch_kind<128>(e.kind, mw, mx, p, e, stages, smem, s); break;
        default: launch_kind<256>(e.kind, mw, mx, p, e, stages, smem, s); break;
    }
}

template <>
void GemmTC<float>::run(const float *, int, int, const float *, int, int, const Epi<float> &, cudaStream_t) {}

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
