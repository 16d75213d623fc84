// pass_program.h -- a bf16 decode pass as a program of projections.
//
// The drafter and verify passes of a bf16 model are built once per batch size
// as a list of projections with their fused epilogues (folded RMSNorms: each
// projection scales its accumulator by the row scale the previous epilogue's
// per-tile sums of squares give).  The host runs the list one kernel per
// projection, attention in between; with DFLASH_DEP_COUNTERS=1 consecutive
// kernels of a pass wait on device completion counters instead of the grid
// release.
#pragma once

#include <vector>

#include "gemm_tc.h"

namespace dfl {

struct PassOp {
    int kind;                  // EpiKind
    Epi<bf16> e;
};

// Raw operands of one op.
struct HostOp {
    const void *W;
    int N, K;
    const void *X;
    int ldx, M;
};

struct PassProgram {
    std::vector<PassOp> ops;
    std::vector<HostOp> hops;        // raw operands of ops[i]
    int key = -1;                    // batch size the program was built for
    // completion counters [2 * n_ops] (projection i: i; attention of layer l:
    // n_ops + l), runs of the program since its counters were cleared, CTAs
    // each counter receives per run, last counter of the pass
    int *d_dep = nullptr;
    unsigned dep_run = 0;
    std::vector<int> dep_ctas;
    int dep_prev = -1;
};

}  // namespace dfl
