// gemm_tc.h -- tensor-core (tcgen05) weight-streaming projection for bf16 models.
#pragma once

#include <string>

#include "kernels.h"

namespace dfl {

int gemm_tc_workspace_floats(int max_rows, int max_n);
int gemm_tc_semaphores();

template <typename T>
struct GemmTC {
    std::string err;
    int init(float *ws, int ws_floats, int *sem, int n_sem) {
        (void)ws; (void)ws_floats; (void)sem; (void)n_sem;
        return 0;
    }
    bool supports(int M, int N, int K) const { (void)M; (void)N; (void)K; return false; }
    void run(const T *X, int ldx, int M, const T *W, int N, int K, const Epi<T> &e, cudaStream_t s) {
        (void)X; (void)ldx; (void)M; (void)W; (void)N; (void)K; (void)e; (void)s;
    }
};

template <typename T>
bool moe_tc_supported() { return false; }

template <typename T>
void run_moe_tc(const T *m, int ldm, int R, int k, const int *sel, const T *w_gate_up, const T *w_down, int H,
                int Fe, int E, T *h, float *part, GemmTC<T> &tc, cudaStream_t s) {
    (void)m; (void)ldm; (void)R; (void)k; (void)sel; (void)w_gate_up; (void)w_down; (void)H; (void)Fe; (void)E;
    (void)h; (void)part; (void)tc; (void)s;
}

}  // namespace dfl
