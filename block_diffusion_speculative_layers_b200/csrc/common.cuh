// common.cuh -- types and small device helpers shared by the DFlash kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

typedef __nv_bfloat16 bf16;

namespace dfl {

// Per-row metadata of one forward pass.
//  target / drafter block rows: seq = slot, pos = absolute position,
//    nk = number of visible keys (causal: pos+1; drafter block: p+B),
//    aux = destination row in the tap buffer (target rows).
//  drafter context rows: seq, pos = context position, aux = 1 if the row is a
//    committed position whose context K/V must be written, else 0.
struct RowMeta {
    int32_t seq, pos, nk, aux;
};

// Device-resident state of one sequence slot.
struct SeqState {
    int32_t len;        // valid target KV positions == position of the anchor
    int32_t anchor;     // last committed token (input of the next block's row 0)
    int32_t ctx_len;    // valid drafter context positions
    int32_t pend_pos0;  // first position of context rows still to be injected
    int32_t pend_n;     // number of such rows (their taps sit in the pending tap rows of the slot)
    int32_t n_out;      // tokens emitted after the prompt (the first comes from prefill)
    int32_t max_new;    // stop after this many tokens
    int32_t done;
};

// Accumulated decode statistics (device side).
struct DevStats {
    unsigned long long iterations;          // sequence-iterations
    unsigned long long tokens;              // tokens emitted by verify/commit
    unsigned long long hist[32];             // accept lengths a (block size <= 32)
    int32_t n_done;                         // sequences that reached max_new
    int32_t status;                         // nonzero: non-finite logits seen
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// Two-plane activations (bf16 models).  A value v of a GEMM input, q or the
// K/V cache is kept as hi = bf16(v) at p[i] and lo = bf16(v - hi) at p[i + lo],
// so hi + lo carries ~16 significant bits while each plane stays a bf16
// tensor-core operand; lo == 0 means a single plane.
template <typename T>
__device__ __forceinline__ void st_act(T *p, size_t i, size_t lo, float v) {
    const T h = from_f<T>(v);
    p[i] = h;
    if (lo) p[i + lo] = from_f<T>(v - to_f(h));
}
template <typename T>
__device__ __forceinline__ float ld_act(const T *p, size_t i, size_t lo) {
    float v = to_f(p[i]);
    if (lo) v += to_f(p[i + lo]);
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// (value, index) max with the lowest index winning exact ties.
__device__ __forceinline__ void argmax_merge(float &v, int &i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

// Commit one block of sequence i (slot s): drafts d[0..a) were accepted and x
// follows them.  Records the committed row (tokens, then -1), emits the tokens
// up to max_new, makes x the next anchor and moves the length and the pending
// drafter-context rows by a + 1; a finished sequence only gets its row.
__device__ __forceinline__ void commit_block(SeqState &S, int s, int i, int a, const int *d, int x, int B,
                                             int *committed, int *out_tok, int out_ld, DevStats *stats) {
    if (committed)
        for (int k = 0; k < B; ++k) committed[i * B + k] = (k < a) ? d[k] : (k == a ? x : -1);
    if (S.done) return;
    int emitted = 0;
    for (int k = 0; k <= a; ++k) {
        const int tok = (k < a) ? d[k] : x;
        if (S.n_out < S.max_new) {
            out_tok[(size_t)s * out_ld + S.n_out] = tok;
            S.n_out++;
            emitted++;
        }
    }
    S.anchor = x;
    if (S.n_out >= S.max_new) {
        S.done = 1;
        S.pend_n = 0;
        if (stats) atomicAdd(&stats->n_done, 1);
    } else {
        S.pend_pos0 = S.len;
        S.pend_n = a + 1;
        S.len += a + 1;
    }
    if (stats) {
        atomicAdd(&stats->iterations, 1ull);
        atomicAdd(&stats->tokens, (unsigned long long)emitted);
        atomicAdd(&stats->hist[a], 1ull);
    }
}

}  // namespace dfl

namespace dfl {

// Programmatic dependent launch: let the next kernel in the stream begin its
// prologue now, and wait here until the previous kernel's writes are visible.
// Both are no-ops for kernels launched without the programmatic attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace dfl
