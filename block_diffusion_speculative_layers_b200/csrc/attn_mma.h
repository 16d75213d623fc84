// attn_mma.h -- tensor-core block attention for bf16 models (split-KV).
#pragma once

#include <algorithm>

#include "kernels.h"

namespace dfl {

// Split-KV scratch: unnormalised partial outputs [parts][hd], (max, sum) [parts][2]
// with parts = (query tile, q head, split, row), and one arrival counter per
// (query tile, kv head).
struct AttnScratch {
    float *o_part = nullptr;
    float *ml_part = nullptr;
    int *sem = nullptr;
    size_t max_parts = 0;
    int n_sem = 0;
    int num_sms = 148;  // SMs of the context's device
};

struct AttnWorkspace {
    size_t max_parts = 0;
};
AttnWorkspace attn_workspace_plan(int max_rows, int nq, int nkv, int max_len, int num_sms);

template <typename T>
bool attn_mma_supported(int hd);

// Completion counters of a decode pass (all null: griddepcontrol.wait and no signal).
struct AttnSync {
    const int *dep_ctr = nullptr;  // wait until *dep_ctr >= dep_target
    int dep_target = 0;
    int *done_ctr = nullptr;       // each CTA adds 1 after its last store
    int *err = nullptr;            // device error word (bit 16: a wait timed out)
};

// rows_per_tile: rows of one sequence that share a query tile (block size for
// draft/verify, 16 for prompt rows, 1 for single-row target steps).
// lo != 0: q, K/V and out are two-plane activations (low plane lo elements on).
// Returns the number of CTAs launched.
template <typename T>
int launch_attention_mma(const T *q, int ldq, const T *kc, const T *vc, const RowMeta *meta, int R, int rows_per_tile,
                         int nq, int nkv, int hd, int max_len, T *out, int ldo, size_t lo, const AttnScratch &ws,
                         cudaStream_t s, const AttnSync &sy = AttnSync());

}  // namespace dfl
