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

template <int HD>
__global__ void __launch_bounds__(256) attn_mma_kernel(const bf16 *__restrict__ q, int ldq, const bf16 *__restrict__ kc,
                                                       const bf16 *__restrict__ vc, const RowMeta *__restrict__ meta,
                                                       int R, int rows_per_tile, int nq, int nkv, int max_len, int chunk,
                                                       int n_splits, float scale_log2, bf16 *__restrict__ out, int ldo,
                                                       float *o_part, float *ml_part, int *sem) {
    constexpr int LDS = HD + 8;  // padded smem row (bf16 elements)
    extern __shared__ __align__(16) uint8_t smem_raw[];
    bf16 *Ks = reinterpret_cast<bf16 *>(smem_raw);  // [2][KB][LDS]
    bf16 *Vs = Ks + 2 * KB * LDS;                    // [2][KB][LDS]
    __shared__ int s_last;

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
    const int kb = split * chunk;
    const int ke = min(kb + chunk, nk_max);

    const size_t head_off = ((size_t)seq * nkv + kvh) * (size_t)max_len * HD;
    const bf16 *Kg = kc + head_off;
    const bf16 *Vg = vc + head_off;

    // Q fragments (A operand, 16 rows x HD)
    uint32_t qa[HD / 16][4];
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const int c0 = kk * 16 + (lane & 3) * 2;
        const bf16 *qa_row = q + (size_t)(r0 + ra) * ldq + h * HD;
        const bf16 *qb_row = q + (size_t)(r0 + rb) * ldq + h * HD;
        qa[kk][0] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0) : 0u;
        qa[kk][1] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0) : 0u;
        qa[kk][2] = ra < nrows ? *reinterpret_cast<const uint32_t *>(qa_row + c0 + 8) : 0u;
        qa[kk][3] = rb < nrows ? *reinterpret_cast<const uint32_t *>(qb_row + c0 + 8) : 0u;
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
            uint32_t pa[4];
            pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
            pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
            pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
            pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < HD / 16; ++dp) {
                // matrices (keys 0-7, d 0-7), (keys 8-15, d 0-7), (keys 0-7, d 8-15), (keys 8-15, d 8-15)
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int dim = dp * 16 + (lane >> 4) * 8;
                uint32_t b0, b1, b2, b3;
                ldm_x4_t(b0, b1, b2, b3, Vt + (size_t)key * LDS + dim);
                mma16816(o[2 * dp], pa, b0, b1);
                mma16816(o[2 * dp + 1], pa, b2, b3);
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
            if (ra < nrows)
                *reinterpret_cast<__nv_bfloat162 *>(out + (size_t)(r0 + ra) * ldo + h * HD + d) =
                    __floats2bfloat162_rn(o[j][0] * ia, o[j][1] * ia);
            if (rb < nrows)
                *reinterpret_cast<__nv_bfloat162 *>(out + (size_t)(r0 + rb) * ldo + h * HD + d) =
                    __floats2bfloat162_rn(o[j][2] * ib, o[j][3] * ib);
        }
        return;
    }
    // partials
    const size_t pbase = ((size_t)(tile * nq + h) * n_splits + split) * 16;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
        const int d = j * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2 *>(o_part + (pbase + ra) * HD + d) = make_float2(o[j][0], o[j][1]);
        *reinterpret_cast<float2 *>(o_part + (pbase + rb) * HD + d) = make_float2(o[j][2], o[j][3]);
    }
    if ((lane & 3) == 0) {
        *reinterpret_cast<float2 *>(ml_part + (pbase + ra) * 2) = make_float2(m_a, l_a);
        *reinterpret_cast<float2 *>(ml_part + (pbase + rb) * 2) = make_float2(m_b, l_b);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int old = atomicAdd(&sem[tile * nkv + kvh], 1);
        s_last = (old == n_splits - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // combine all splits for the group's heads and the tile's rows, in split order
    for (int e = threadIdx.x; e < grp * 16 * HD; e += nthr) {
        const int hh = e / (16 * HD), rem = e % (16 * HD), row = rem / HD, d = rem % HD;
        if (row >= nrows) continue;
        const int hq = kvh * grp + hh;
        const size_t b0 = ((size_t)(tile * nq + hq) * n_splits) * 16 + row;
        float mstar = -INFINITY;
        for (int s2 = 0; s2 < n_splits; ++s2) mstar = fmaxf(mstar, __ldcg(ml_part + (b0 + (size_t)s2 * 16) * 2));
        const float mu = mstar == -INFINITY ? 0.f : mstar;
        float lsum = 0.f, acc = 0.f;
        for (int s2 = 0; s2 < n_splits; ++s2) {
            const size_t bb = b0 + (size_t)s2 * 16;
            const float ms = __ldcg(ml_part + bb * 2), ls = __ldcg(ml_part + bb * 2 + 1);
            const float w = exp2f(ms - mu);
            lsum += ls * w;
            acc += __ldcg(o_part + bb * HD + d) * w;
        }
        out[(size_t)(r0 + row) * ldo + hq * HD + d] = __float2bfloat16_rn(lsum > 0.f ? acc / lsum : 0.f);
    }
    if (threadIdx.x == 0) sem[tile * nkv + kvh] = 0;
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

template <>
void launch_attention_mma<bf16>(const bf16 *q, int ldq, const bf16 *kc, const bf16 *vc, const RowMeta *meta, int R,
                                int rows_per_tile, int nq, int nkv, int hd, int max_len, bf16 *out, int ldo,
                                const AttnScratch &ws, cudaStream_t s) {
    if (R <= 0) return;
    if (!g_num_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int n_tiles = (R + rows_per_tile - 1) / rows_per_tile;
    const int grp = nq / nkv;
    const int ctas = n_tiles * nkv;
    int n_splits = std::max(1, std::min((max_len + 255) / 256, (2 * g_num_sms + ctas - 1) / ctas));
    // partial buffers bound the split count
    while (n_splits > 1 && (size_t)n_tiles * nq * n_splits * 16 > ws.max_parts) --n_splits;
    if ((size_t)n_tiles * nkv > (size_t)ws.n_sem) n_splits = 1;
    int chunk = (max_len + n_splits - 1) / n_splits;
    chunk = (chunk + at::KB - 1) / at::KB * at::KB;
    n_splits = (max_len + chunk - 1) / chunk;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
    dim3 grid(n_tiles, nkv, n_splits);
    const int threads = 32 * grp;
    if (hd == 128) {
        const size_t smem = 2 * 2 * at::KB * (128 + 8) * sizeof(bf16);
        static bool set = false;
        if (!set) {
            cudaFuncSetAttribute(at::attn_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            set = true;
        }
        at::attn_mma_kernel<128><<<grid, threads, smem, s>>>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len,
                                                             chunk, n_splits, scale_log2, out, ldo, ws.o_part,
                                                             ws.ml_part, ws.sem);
    } else {
        const size_t smem = 2 * 2 * at::KB * (64 + 8) * sizeof(bf16);
        static bool set = false;
        if (!set) {
            cudaFuncSetAttribute(at::attn_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            set = true;
        }
        at::attn_mma_kernel<64><<<grid, threads, smem, s>>>(q, ldq, kc, vc, meta, R, rows_per_tile, nq, nkv, max_len,
                                                            chunk, n_splits, scale_log2, out, ldo, ws.o_part,
                                                            ws.ml_part, ws.sem);
    }
}

template <>
void launch_attention_mma<float>(const float *, int, const float *, const float *, const RowMeta *, int, int, int, int,
                                 int, int, float *, int, const AttnScratch &, cudaStream_t) {}

}  // namespace dfl
