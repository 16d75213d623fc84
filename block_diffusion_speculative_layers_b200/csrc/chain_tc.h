// chain_tc.h -- persistent projection chain for bf16 decode passes.
//
// One launch executes a run of dependent projections (e.g. O -> gate/up ->
// down -> next layer's QKV) on one CTA per SM.  The TMA ring of every CTA
// streams the next projection's weights while the current one finishes: only
// the activation loads of projection j wait, on a device-side completion
// counter, until every CTA has finished the epilogue of projection j-1.
#pragma once

#include <cuda.h>

#include <string>
#include <vector>

#include "gemm_tc.h"

namespace dfl {

struct ChainOp {
    int kind;                  // EpiKind
    TcParams p;                // M, N, K, n_tiles, m_tiles (1), k_steps, splits, swiglu_F, lm_part, keep_logits
    const CUtensorMap *wmap;   // device address of the weight tensor map
    const CUtensorMap *xmap;   // device address of the activation tensor map
    Epi<bf16> e;
    float *ws;                 // partial tiles: slot tinfo[t].z + part -> [TM][128] floats
    int *tile_cnt;             // [tiles] arrival counters (monotonic across launches)
    const int4 *tinfo;         // per tile: (first CTA covering it, number of CTAs covering it, first slot, 0)
};

struct ChainLaunch {
    const ChainOp *ops;        // device array of the program
    int op_begin, op_end;      // ops executed by this launch
    unsigned epoch;            // how many times the program has run, including this one
    int *op_done;              // [n_ops] completion counters (monotonic)
    int *err;
    int stages;
    int planes;                // activation planes of every op (2: hi + lo)
};

// Raw operands of one op, for running a program one kernel per projection.
struct HostOp {
    const void *W;
    int N, K;
    const void *X;
    int ldx, M;
};

// Host-side program: a list of projections uploaded once, launched in runs
// (persistent chains) or one kernel per projection (same epilogues).
struct ChainProgram {
    std::vector<ChainOp> ops;
    std::vector<HostOp> hops;        // raw operands of ops[i]
    std::vector<CUtensorMap> maps;   // uploaded next to the ops
    ChainOp *d_ops = nullptr;        // device copies (state arena)
    CUtensorMap *d_maps = nullptr;
    int *d_op_done = nullptr;
    int *d_tile_cnt = nullptr;
    int4 *d_tinfo = nullptr;
    std::vector<int4> tinfo;     // host copy, uploaded next to the ops
    float *d_ws = nullptr;           // two split-K partial buffers (op parity)
    size_t ws_floats = 0;            // floats per buffer
    int tm = 16;
    int planes = 1;
    unsigned epoch = 0;
    int key = -1;                    // program identity (pass, batch) it was built for
    bool valid = true;               // false: the shapes do not fit the reserved workspace
    // per-kernel execution: completion counters [2 * n_ops] (projection i: i;
    // attention of layer l: n_ops + l), runs of the program since its counters
    // were cleared, CTAs each counter receives per run, last counter of the pass
    int *d_dep = nullptr;
    unsigned dep_run = 0;
    std::vector<int> dep_ctas;
    int dep_prev = -1;
};

// Launch ops [b, e) of a program (epoch must already be advanced for this run).
void launch_chain(const ChainProgram &prog, int b, int e, int num_sms, int *err, cudaStream_t s);
int chain_stages(int tm, int planes);
size_t chain_smem_bytes(int tm, int planes, int stages);

}  // namespace dfl
