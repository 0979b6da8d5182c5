// norm.cuh - one sum of squares per token for the RMSNorm row scales.
//
// When the residual projections run on the CTA-pair pipeline they leave one
// partial sum of squares per 32 features and token ([d / 32, M]).  Every
// consumer of the norm would otherwise add all of them up for each tile it
// scales.  This kernel adds them once per token, in index order (the order
// the consumers use, sixteen loads in flight), and stores the total in the
// first partial's place: a consumer told to read one partial gets the same
// bits as from all of them.
#pragma once

#include "dg_common.cuh"

namespace dg {
namespace norm {

constexpr int COLLAPSE_THREADS = 256;

// ssq [n, M] in place: ssq[0, t] = sum_q ssq[q, t].  One thread per token
// (a thread touches only its own column).
__global__ void __launch_bounds__(COLLAPSE_THREADS)
    ssq_collapse_kernel(float* __restrict__ ssq, int n, int M) {
  griddep_wait();
  griddep_launch();
  const int t = static_cast<int>(blockIdx.x) * COLLAPSE_THREADS + static_cast<int>(threadIdx.x);
  if (t >= M) return;
  float acc = 0.f;
  for (int q0 = 0; q0 < n; q0 += 16) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = q0 + j < n ? ssq[static_cast<size_t>(q0 + j) * M + t] : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) acc += v[j];
  }
  ssq[t] = acc;
}

}  // namespace norm
}  // namespace dg
