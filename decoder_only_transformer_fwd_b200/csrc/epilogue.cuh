// Element-wise GEMM epilogues shared by the CUDA-core and tcgen05 GEMMs.
//
// The block structure is "The Mathematics of Karpathy's nanochat",
// §Residual Stream with Learnable Scalars: x <- lam x + mu x0 before each
// block, x <- x + Attn(.), x <- x + MLP(.); backout ("nanochat depth sweep"
// card, Architecture list) subtracts beta times the captured block output
// before the final norm.  The MLP activation is ReLU^2 (§Feed-Forward
// Network) and the logits are soft-capped (§Logit Softcap).
#pragma once

#include "nc_internal.cuh"

namespace nc {

template <typename T>
__device__ __forceinline__ void epi_apply(const EpiParams& ep, int m, int n, float acc) {
  switch (ep.mode) {
    case EPI_STORE:
      Act<T>::st(reinterpret_cast<T*>(ep.out) + (size_t)m * ep.ldo + n, acc);
      break;
    case EPI_RELU2: {
      const float r = fmaxf(acc, 0.f);
      Act<T>::st(reinterpret_cast<T*>(ep.out) + (size_t)m * ep.ldo + n, r * r);
    } break;
    case EPI_RESID:
      ep.x[(size_t)m * ep.ldx + n] += acc;
      break;
    case EPI_BLOCK_END: {
      const size_t i = (size_t)m * ep.ldx + n;
      float v = ep.x[i] + acc;
      if (ep.capture_bo) ep.xbo[i] = v;
      if (ep.end_kind == 1)
        v = (*ep.lam) * v + (*ep.mu) * ep.x0[i];
      else if (ep.end_kind == 2)
        v = v - ep.beta * ep.xbo[i];
      ep.x[i] = v;
    } break;
    case EPI_SOFTCAP:
      if (n < ep.vocab) ep.logits[(size_t)m * ep.ldl + n] = ep.cap * tanhf(acc / ep.cap);
      break;
    default:
      break;
  }
}

}  // namespace nc
