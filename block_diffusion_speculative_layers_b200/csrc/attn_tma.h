// attn_tma.h -- latency-oriented block attention for bf16 models: K/V tiles
// by TMA through an mbarrier ring, keys split over a thread-block cluster.
#pragma once

#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "kernels.h"

namespace dfl {

struct AttnTmaArgs {
    const bf16 *q = nullptr;  // [R][ldq], q head h at columns h*hd (low plane lo elements on)
    int ldq = 0;
    const RowMeta *meta = nullptr;  // per row: sequence slot, position, visible keys nk
    int R = 0, rows_per_tile = 16, nq = 0, nkv = 0, max_len = 0;
    int n_seq = 0;                  // sequence slots of the K/V caches
    int one_seq = 0;                // 1: every row is of one sequence (a prefill chunk)
    int layer = 0;                  // layer of the K/V maps
    float scale_log2 = 0.f;         // log2(e) / sqrt(hd)
    bf16 *out = nullptr;            // [R][ldo] (low plane lo elements on)
    int ldo = 0;
    size_t lo = 0;                  // two-plane activations: low plane offset (elements), 0: one plane
    int *err = nullptr;             // device error word (bit 32: a bounded wait expired)
    int n_splits = 1, stages = 3;   // set by the launcher
    // completion counters (decode passes): wait until *dep_ctr >= dep_target instead
    // of griddepcontrol.wait (nullptr: griddepcontrol.wait); each CTA adds 1 to
    // *done_ctr after its last store (nullptr: no signal)
    const int *dep_ctr = nullptr;
    int dep_target = 0;
    int *done_ctr = nullptr;
};

bool attn_tma_supported(int hd, int grp);

// Tensor map of one model's K (or V) cache [layer][seq][kv head][max_len][hd]
// viewed as (hd, position, seq * kv head, layer[, plane]): 4-D for one plane,
// 5-D with the low plane `lo` elements on; box {64, kt, 1, 1[, 2]}, 128-byte
// swizzle.  false if the driver cannot encode it.
bool attn_tma_make_map(CUtensorMap *map, const bf16 *cache, int hd, int max_len, int n_seq_heads, int n_layers,
                       size_t layer_elems, size_t lo, int kt);

// The K and V maps of one model's caches, with 16- and 32-key boxes.
struct AttnTmaMaps {
    CUtensorMap k16, v16, k32, v32;
};

// q heads per CTA and keys per tile the launcher picks for n_tiles query tiles of
// a GQA group size grp (one_seq: the tiles are one sequence's prefill chunk)
int attn_tma_hpc(int grp, int n_tiles, int nkv, int num_sms, bool one_seq);
int attn_tma_kt(int hpc);

// Launch on stream s; returns the CTAs launched, -1 if the launch failed.
int launch_attention_tma(const AttnTmaMaps &maps, AttnTmaArgs a, int hd, bool split, int num_sms, cudaStream_t s);

}  // namespace dfl
