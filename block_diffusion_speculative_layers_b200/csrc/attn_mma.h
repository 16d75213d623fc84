// attn_mma.h -- tensor-core attention for bf16 models.
#pragma once

#include "kernels.h"

namespace dfl {

template <typename T>
bool attn_mma_supported(int hd) { (void)hd; return false; }

template <typename T>
void launch_attention_mma(const T *q, int ldq, const T *kc, const T *vc, const RowMeta *meta, int R, int nq, int nkv,
                          int hd, int max_len, T *out, int ldo, cudaStream_t s) {
    (void)q; (void)ldq; (void)kc; (void)vc; (void)meta; (void)R; (void)nq; (void)nkv; (void)hd; (void)max_len;
    (void)out; (void)ldo; (void)s;
}

}  // namespace dfl
