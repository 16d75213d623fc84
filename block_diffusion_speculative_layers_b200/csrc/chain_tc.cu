// chain_tc.cu -- persistent chain of dependent tensor-core projections.
//
// Per CTA (one per SM, 192 threads, the roles of gemm_tc.cu):
//   warp 0      one thread streams the TMA ring over every (op, unit, k-step)
//               this CTA owns, in order.  Weight boxes are issued as soon as a
//               ring slot is free; the activation box of op j is issued only
//               once every CTA has finished op j-1 (device completion counter,
//               acquire) -- until then it waits in a small queue while the
//               weights of op j keep streaming;
//   warp 1      TMEM (two accumulators) + tcgen05.mma issue;
//   warps 2..5  epilogue per unit; K-split units park their partial tile in
//               global memory and the last-arriving CTA of a tile sums the
//               partials in split order (deterministic) and runs the fused
//               epilogue; after its last unit of op j a CTA bumps op_done[j].
// Work split (stream-K): the n_tiles * k_steps (tile, k-step) pairs of an op
// are cut into gridDim.x equal contiguous ranges, one per CTA, so every CTA
// streams the same number of weight bytes; a range covers whole or partial
// tiles.  A tile covered by several CTAs is reduced by the last one to arrive,
// summing the parked partials in k order (deterministic).  Every wait is
// bounded (2 s); on expiry an error bit is set.
#include <algorithm>
#include <cstring>

#include "chain_tc.h"
#include "launch.h"
#include "tc_device.cuh"

namespace dfl {
namespace tc {

struct PendingX {
    int s, j, k;
};

// This CTA's contiguous share [s0, s1) of the op's tile-k-steps.  Ops with
// fewer tile-k-steps than CTAs are dealt to the first `total` CTAs only.
__device__ __forceinline__ void cta_range(const ChainOp &op, int b, int G, long long &s0, long long &s1) {
    const long long total = (long long)op.p.n_tiles * op.p.k_steps;
    const long long g = total < G ? total : G;
    if (b >= g) {
        s0 = s1 = 0;
        return;
    }
    s0 = total * b / g;
    s1 = total * (b + 1) / g;
}

template <int TM>
__global__ void __launch_bounds__(NT, 1) chain_kernel(ChainLaunch L) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int B_BYTES = TM * 128 * L.planes;
    const bool wide = L.planes == 2 && TM <= 128;  // one N = 2*TM MMA over both planes
    const int lo_col = wide ? TM : 0;
    const int NC1 = max(32, wide ? 2 * TM : TM);
    const int stages = L.stages;
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)stages * A_BYTES;
    float *stg = (float *)(sB + (size_t)stages * B_BYTES);
    float2 *red = (float2 *)(stg + 128 * STG_LD);
    RowMeta *smeta = (RowMeta *)(red + 4 * CH);
    float *rsc = (float *)(smeta + CH);       // [RS_MAX] row scales of the folded norm
    uint64_t *full = (uint64_t *)(rsc + RS_MAX);
    uint64_t *empty = full + stages;
    uint64_t *acc_full = empty + stages;   // [2]
    uint64_t *acc_empty = acc_full + 2;    // [2]
    uint32_t *tmem_slot = (uint32_t *)(acc_empty + 2);
    int *flag = (int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int target = (int)L.epoch * G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        mbar_init(&acc_empty[0], 4);
        mbar_init(&acc_empty[1], 4);
        flag[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(2 * NC1));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            const uint64_t wpol = l2_evict_first_policy();
            PendingX pend[16];
            int np = 0, ready_upto = L.op_begin - 1, it = 0;
            bool abort = false;
            auto x_ready = [&](int j) -> bool {  // non-blocking
                if (j <= ready_upto) return true;
                if (j == L.op_begin) return false;  // needs griddepcontrol.wait (blocking)
                if (ld_acquire(&L.op_done[j - 1]) >= target) {
                    fence_proxy_async_global();
                    ready_upto = j;
                    return true;
                }
                return false;
            };
            auto wait_ready = [&](int j) -> bool {  // blocking, bounded
                if (j <= ready_upto) return true;
                if (j == L.op_begin) {
                    pdl_wait();
                } else if (!wait_counter(&L.op_done[j - 1], target, L.err)) {
                    return false;
                }
                fence_proxy_async_global();
                ready_upto = j;
                return true;
            };
            auto issue_x = [&](const PendingX &px) {
                if (L.planes == 2) tma_load_3d(sB + (size_t)px.s * B_BYTES, L.ops[px.j].xmap, px.k, 0, 0, &full[px.s]);
                else tma_load_2d(sB + (size_t)px.s * B_BYTES, L.ops[px.j].xmap, px.k, 0, &full[px.s]);
            };
            auto flush = [&](bool block) -> bool {
                int i = 0;
                for (; i < np; ++i) {
                    const bool ok = block ? wait_ready(pend[i].j) : x_ready(pend[i].j);
                    if (!ok) {
                        if (block) return false;
                        break;
                    }
                    issue_x(pend[i]);
                }
                for (int t = i; t < np; ++t) pend[t - i] = pend[t];
                np -= i;
                return true;
            };
            for (int j = L.op_begin; j < L.op_end && !abort; ++j) {
                const ChainOp &op = L.ops[j];
                const int ks = op.p.k_steps;
                long long g0, g1;
                cta_range(op, blockIdx.x, G, g0, g1);
                for (long long g = g0; g < g1 && !abort;) {
                    const int nt = (int)(g / ks);
                    const int kb = (int)(g - (long long)nt * ks);
                    const int ke = (int)min((long long)ks, g1 - (long long)nt * ks);
                    g = (long long)nt * ks + ke;
                    const int rowA0 = op.p.swiglu_F ? nt * 64 : nt * 128;
                    const int rowA1 = op.p.swiglu_F ? op.p.swiglu_F + nt * 64 : nt * 128 + 64;
                    for (int kk = kb; kk < ke; ++kk, ++it) {
                        const int s = it % stages;
                        if (it >= stages) {
                            const uint32_t par = ((it / stages) & 1) ^ 1;
                            if (!mbar_try(&empty[s], par)) {
                                // the ring is full: queued activation loads must go out before blocking
                                if (np > 0 && !flush(true)) {
                                    abort = true;
                                    break;
                                }
                                if (!mbar_wait(&empty[s], par, L.err)) {
                                    abort = true;
                                    break;
                                }
                            }
                        }
                        uint8_t *a = sA + (size_t)s * A_BYTES;
                        mbar_expect_tx(&full[s], A_BYTES + B_BYTES);
                        tma_load_2d_hint(a, op.wmap, kk * BK, rowA0, &full[s], wpol);
                        tma_load_2d_hint(a + A_BYTES / 2, op.wmap, kk * BK, rowA1, &full[s], wpol);
                        const PendingX px{s, j, kk * BK};
                        if (np == 0 && x_ready(j)) issue_x(px);
                        else pend[np++] = px;
                        if (np > 0) flush(false);
                    }
                }
            }
            if (!abort && np > 0) flush(true);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_bf16(wide ? 2 * TM : TM);
            int it = 0, lt = 0;
            bool ok = true;
            for (int j = L.op_begin; j < L.op_end && ok; ++j) {
                const ChainOp &op = L.ops[j];
                const int ks = op.p.k_steps;
                long long g0, g1;
                cta_range(op, blockIdx.x, G, g0, g1);
                for (long long g = g0; g < g1 && ok; ++lt) {
                    const int nt = (int)(g / ks);
                    const int kb = (int)(g - (long long)nt * ks);
                    const int ke = (int)min((long long)ks, g1 - (long long)nt * ks);
                    g = (long long)nt * ks + ke;
                    const int b = lt & 1;
                    if (lt >= 2 && !mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1, L.err)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t acc = tmem + (uint32_t)(b * NC1);
                    for (int kk = kb; kk < ke; ++kk, ++it) {
                        const int s = it % stages;
                        if (!mbar_wait(&full[s], (it / stages) & 1, L.err)) {
                            ok = false;
                            break;
                        }
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        const uint64_t da = sw128_desc(smem_u32(sA + (size_t)s * A_BYTES));
                        const uint64_t db = sw128_desc(smem_u32(sB + (size_t)s * B_BYTES));
#pragma unroll
                        for (int k4 = 0; k4 < BK / 16; ++k4) {
                            mma_bf16(acc, da + (uint64_t)(k4 * 2), db + (uint64_t)(k4 * 2), idesc,
                                     (kk > kb || k4 > 0) ? 1u : 0u);
                            if (L.planes == 2 && !wide)  // lo plane, TM rows further on
                                mma_bf16(acc, da + (uint64_t)(k4 * 2), db + (uint64_t)((TM * 128) >> 4) + (uint64_t)(k4 * 2),
                                         idesc, 1u);
                        }
                        mma_commit(&empty[s]);
                    }
                    mma_commit(&acc_full[b]);
                }
            }
        }
    } else {
        // ---------------- epilogue warps 2..5 ----------------
        pdl_wait();
        const int q = warp & 3;
        const int n_local = q * 32 + lane;
        int lt = 0;
        for (int j = L.op_begin; j < L.op_end; ++j) {
            const ChainOp &op = L.ops[j];
            if (j > L.op_begin) {
                // every CTA has finished op j-1 (normally long since true)
                if (threadIdx.x == 64) wait_counter(&L.op_done[j - 1], target, L.err);
                epi_bar();
            }
            if (op.e.rs_ssq) all_row_scales(op.e, 0, TM, op.p.M, rsc);
            const int ks = op.p.k_steps;
            long long g0, g1;
            cta_range(op, blockIdx.x, G, g0, g1);
            for (long long g = g0; g < g1; ++lt) {
                const int nt = (int)(g / ks);
                const int ke = (int)min((long long)ks, g1 - (long long)nt * ks);
                g = (long long)nt * ks + ke;
                const int4 ti = op.tinfo[nt];  // first CTA, CTAs covering the tile, first slot
                const int S = ti.y;
                const int sp = (int)blockIdx.x - ti.x;
                const int b = lt & 1;
                const uint32_t trow = tmem + (uint32_t)(b * NC1) + ((uint32_t)(q * 32) << 16);
                const bool ok = mbar_wait(&acc_full[b], (lt >> 1) & 1, L.err);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                float v[CH];
                if (S == 1) {
                    for (int c = 0; c < TM; c += CH) {
                        if (ok) acc_ld16(trow, c, lo_col, v);
                        else
#pragma unroll
                            for (int jj = 0; jj < CH; ++jj) v[jj] = 0.f;
                        if (c == TM - CH) {
                            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&acc_empty[b]);
                        }
                        switch (op.kind) {
                            case EPI_QKV: epilogue_chunk<EPI_QKV>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            case EPI_RESID: epilogue_chunk<EPI_RESID>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            case EPI_SWIGLU: epilogue_chunk<EPI_SWIGLU>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            case EPI_LOGITS: epilogue_chunk<EPI_LOGITS>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            case EPI_NORMOUT: epilogue_chunk<EPI_NORMOUT>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            default: epilogue_chunk<EPI_STORE>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                        }
                    }
                } else {
                    float *mine = op.ws + ((size_t)ti.z + sp) * (size_t)TM * 128;
                    for (int c = 0; c < TM; c += CH) {
                        if (ok) acc_ld16(trow, c, lo_col, v);
                        else
#pragma unroll
                            for (int jj = 0; jj < CH; ++jj) v[jj] = 0.f;
                        if (c == TM - CH) {
                            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&acc_empty[b]);
                        }
#pragma unroll
                        for (int jj = 0; jj < CH; ++jj) mine[(size_t)(c + jj) * 128 + n_local] = v[jj];
                    }
                    __threadfence();
                    epi_bar();
                    if (threadIdx.x == 64) {
                        const int old = atomicAdd(&op.tile_cnt[nt], 1);
                        flag[0] = (old == (int)L.epoch * S - 1) ? 1 : 0;
                    }
                    epi_bar();
                    if (flag[0]) {
                        __threadfence();
                        const float *base = op.ws + (size_t)ti.z * TM * 128;
                        for (int c = 0; c < TM; c += CH) {
#pragma unroll
                            for (int jj = 0; jj < CH; ++jj) v[jj] = 0.f;
                            for (int s2 = 0; s2 < S; ++s2) {
                                float t[CH];
                                const float *src = base + ((size_t)s2 * TM + c) * 128 + n_local;
#pragma unroll
                                for (int jj = 0; jj < CH; ++jj) t[jj] = __ldcg(src + (size_t)jj * 128);
#pragma unroll
                                for (int jj = 0; jj < CH; ++jj) v[jj] += t[jj];
                            }
                            switch (op.kind) {
                                case EPI_QKV: epilogue_chunk<EPI_QKV>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                                case EPI_RESID: epilogue_chunk<EPI_RESID>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                                case EPI_SWIGLU: epilogue_chunk<EPI_SWIGLU>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                                case EPI_LOGITS: epilogue_chunk<EPI_LOGITS>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                                case EPI_NORMOUT: epilogue_chunk<EPI_NORMOUT>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                                default: epilogue_chunk<EPI_STORE>(op.p, op.e, nt, n_local, q, lane, c, CH, v, stg, red, smeta, rsc + c); break;
                            }
                        }
                    }
                    epi_bar();  // flag[0] is rewritten by the next unit
                }
            }
            // this CTA's share of op j is written: every writer fences (generic and
            // async proxy, GPU scope), then one thread publishes it (release)
            __threadfence();
            fence_proxy_async_global();
            epi_bar();
            if (threadIdx.x == 64) {
                __threadfence();
                atomicAdd(&L.op_done[j], 1);
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * NC1));
    }
}

}  // namespace tc

static size_t chain_fixed_bytes() {
    return 1024 + 128 * tc::STG_LD * 4 + 4 * tc::CH * 8 + tc::CH * 16 + tc::RS_MAX * 4 + 64 * 8 + 64;
}

int chain_stages(int tm, int planes) {
    // ~150 KB keeps room on each SM for an attention CTA (~70 KB) of the next kernel
    const size_t budget = tm <= 32 ? 150 * 1024 : 200 * 1024;
    const size_t stage = tc::A_BYTES + (size_t)tm * 128 * planes;
    return (int)std::max<size_t>(2, std::min<size_t>(16, (budget - chain_fixed_bytes()) / stage));
}

size_t chain_smem_bytes(int tm, int planes, int stages) {
    return chain_fixed_bytes() + (size_t)stages * (tc::A_BYTES + (size_t)tm * 128 * planes);
}

template <int TM>
static void launch_tm(const ChainLaunch &L, int num_sms, size_t smem, cudaStream_t s) {
    static bool set = false;
    if (!set) {
        cudaFuncSetAttribute(tc::chain_kernel<TM>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        set = true;
    }
    launch_k(tc::chain_kernel<TM>, dim3(num_sms), dim3(tc::NT), smem, s, 1, L);
}

void launch_chain(const ChainProgram &prog, int b, int e, int num_sms, int *err, cudaStream_t s) {
    ChainLaunch L;
    L.ops = prog.d_ops;
    L.op_begin = b;
    L.op_end = e;
    L.epoch = prog.epoch;
    L.op_done = prog.d_op_done;
    L.err = err;
    L.planes = prog.planes;
    L.stages = chain_stages(prog.tm, prog.planes);
    const size_t smem = chain_smem_bytes(prog.tm, prog.planes, L.stages);
    switch (prog.tm) {
        case 16: launch_tm<16>(L, num_sms, smem, s); break;
        case 32: launch_tm<32>(L, num_sms, smem, s); break;
        case 64: launch_tm<64>(L, num_sms, smem, s); break;
        case 128: launch_tm<128>(L, num_sms, smem, s); break;
        default: launch_tm<256>(L, num_sms, smem, s); break;
    }
}

}  // namespace dfl
