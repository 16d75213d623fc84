// gemm_tc.h -- tensor-core (tcgen05 + TMEM + TMA) weight-streaming projection
// for bf16 models.
//
// Y[M][N] = X[M][K] . W[N][K]^T is computed "swap-AB": the weight tile is the
// 128-row A operand and the few activation rows (M = batch x block) are the
// N operand of tcgen05.mma, so a 16-row decode step still runs on the tensor
// cores while W streams through shared memory exactly once.
#pragma once

#include <cuda.h>

#include <string>
#include <unordered_map>

#include "kernels.h"

namespace dfl {

int gemm_tc_workspace_floats(int max_rows, int max_n);
int gemm_tc_semaphores();

// Launch parameters shared by host and device.
struct TcParams {
    int M, N, K;            // logical sizes (N = 2F for SwiGLU)
    int n_tiles, m_tiles;   // tiles of 128 weight rows (64 output columns for SwiGLU) x TM rows
    int k_steps, splits;    // 64-wide K steps in total; K splits
    int swiglu_F;           // SwiGLU: rows [0,F) gate, [F,2F) up; else 0
    float *ws;              // split-K partials
    int *sem;               // per-tile arrival counters (self-resetting)
    int *err;               // device error word (bounded waits)
    float2 *lm_part;        // EPI_LOGITS: per (n_tile, row) best (value, index)
    int keep_logits;        // EPI_LOGITS: also store fp32 logits in Y
    int planes;             // activation planes (2: hi + lo, two MMAs per K step)
    // completion counters (decode passes): wait until *dep_ctr >= dep_target instead
    // of griddepcontrol.wait (dep_ctr == nullptr: griddepcontrol.wait); each CTA adds
    // 1 to *done_ctr after its last store (done_ctr == nullptr: no signal)
    const int *dep_ctr;
    int dep_target;
    int *done_ctr;
    const float *w_scale;   // FP8 weights: fp32 scale of every weight row (the codes' row of W)
    // FP4 (MXFP4) weights (w_bexp != nullptr): W holds packed E2M1 codes; the
    // exponent bytes of row r's 32-value blocks k/32 = 4j .. 4j+3 are the word
    // w_bexp[j * bs_rows + bs_row0 + r] (UE8M0, byte b = block 4j + b)
    const uint32_t *w_bexp;
    int bs_rows, bs_row0;
    int a_tx;               // FP4: bytes a weight stage's TMA completes (the packed bytes it reads)
    // grouped (MoE experts): blockIdx.y = touched-expert slot, blockIdx.z = row tile of
    // that expert; its rows are g_off[e] .. g_off[e+1]-1 of X (expert-grouped order) and
    // its weights rows e*g_wrows .. of W; nullptr g_off = an ordinary projection
    const int *g_off, *g_touched, *g_list;
    int g_wrows;
};

// Tiling of one projection launch (GemmTC::plan).
struct TcPlan {
    int TM, n_tiles, m_tiles, k_steps, kstep, splits, stages;
    size_t smem;
};

template <typename T>
struct GemmTC {
    std::string err;
    bool failed = false;  // a launch was dropped (tensor map encoding failed); err says why
    bool supports(int M, int N, int K) const;
    int init(float *ws, int ws_floats, int *sem, int n_sem);
    // returns the number of CTAs launched (the count a completion counter reaches per run).
    // W: bf16 [N][K], or with w_scale != nullptr FP8 E4M3 codes [N][K] (one byte each)
    // whose row n stands for w_scale[n] * code value, or with w_bexp != nullptr as
    // well MXFP4 codes [N][K/2] (two E2M1 codes a byte, the low nibble first) whose
    // element (n, k) stands for w_scale[n] * 2^(e - 127) * code value, e the byte
    // (k / 32) % 4 of word (k / 128) * bs_rows + bs_row0 + n of w_bexp.
    int run(const T *X, int ldx, int M, const void *W, int N, int K, const Epi<T> &e, cudaStream_t s,
            const int *dep_ctr = nullptr, int dep_target = 0, int *done_ctr = nullptr,
            const float *w_scale = nullptr, const uint8_t *w_bexp = nullptr, int bs_rows = 0, int bs_row0 = 0);
    // Grouped projection over the touched experts of a MoE layer: W is [E][wrows][K],
    // X the pair rows in expert-grouped order (off[E+1], touched[E] as bucketed),
    // at most max_rows rows per expert.  EPI_SWIGLU writes h in grouped order;
    // EPI_STORE writes row list[pos] of Y.  Returns the CTAs launched.
    int run_grouped(const T *X, int ldx, int n_pairs, const T *W, int wrows, int N, int K, const Epi<T> &e,
                    const int *off, const int *touched, const int *list, int E, int max_rows, cudaStream_t s);
    // tiling of a launch of M activation rows (planes 1 or 2) against an N x K weight
    // matrix (SwiGLU: F output columns, N = 2F), bf16 or FP8
    TcPlan plan(int M, int N, int K, int kind, int F, bool f8, int planes, bool f4 = false) const;
    // LM-head partial argmax buffer (value, index as float bits), [n_tiles][rows]
    void set_lm_part(float2 *p, int cap) { lm_part = p; lm_cap = cap; }
    void set_err(int *e) { err_word = e; }
    float2 *lm_part = nullptr;
    int lm_cap = 0;
    int keep_logits = 0;
    float *ws = nullptr;
    int ws_floats = 0;
    int *sem = nullptr;
    int n_sem = 0;
    int *err_word = nullptr;
    int num_sms = 148;
    // tuning overrides (0 = automatic): K splits per tile, shared-memory budget in KB
    // of unsplit / K-split launches, CTAs per SM the K split aims to fill
    int tune_splits = 0, tune_smem_kb = 0, tune_split_smem_kb = 0, tune_ctas_per_sm = 0;
    int tune_tm_max = 0;  // cap on the activation rows of one tile (more row tiles, weights re-read from L2)
    // FP8 projections: MX planes of the activation rows (codes [planes][mx_mpad][mx_kpad],
    // scale words [K/128][planes][mx_mpad]; every scale byte starts as 127), owned by the caller
    uint8_t *mx_codes = nullptr, *mx_words = nullptr;
    int mx_mpad = 0, mx_kpad = 0;
    const CUtensorMap *mx_map_codes(int M, int K, int tm);
    const CUtensorMap *mx_map_words(int M, int K, int tm);
    std::unordered_map<std::string, CUtensorMap> maps;
    // 2-D map of a [rows][cols] bf16 matrix (leading dimension ld), box {64, box_rows};
    // plane_stride > 0: 3-D map over the hi plane and the lo plane plane_stride
    // elements after it, box {64, box_rows, 2}
    const CUtensorMap *tensor_map(const void *ptr, int rows, int cols, int ld, int box_rows, size_t plane_stride = 0,
                                  bool fp8 = false);
    // 2-D map of [rows][cols] packed E2M1 codes (cols / 2 bytes a row), box {128, box_rows}:
    // each 16 codes (8 bytes) land in 16 bytes of shared memory, the layout the
    // block-scaled MMA reads 4-bit elements in
    const CUtensorMap *fp4_map(const void *ptr, int rows, int cols, int box_rows);
};

// Row-wise argmax over the LM-head partials: mode 0 idx[r]; mode 1 drafter rows.
void launch_lm_argmax(const float2 *part, int n_tiles, int R, int mode, int B, int *idx, DevStats *stats,
                      cudaStream_t s);

template <typename T>
bool moe_tc_supported();

template <typename T>
void run_moe_tc(const T *m, int ldm, int R, int k, const int *sel, const T *w_gate_up, const T *w_down, int H,
                int Fe, int E, T *h, float *part, GemmTC<T> &tc, cudaStream_t s);

}  // namespace dfl
