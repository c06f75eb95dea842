// Offline weight preparation: argument block, scratch layout and entry point.
#pragma once
#include "kq_internal.cuh"

namespace kq {

enum class PrepStatus { Ok, Cuda, Solver };

struct PrepareArgs {
  int K, N, rank, kind;
  bool center;
  const void* W;              // device bf16 [K, N]
  void* weights;              // device, WeightsLayout::total bytes
  void* ws;                   // device scratch, PrepareWs::total bytes
  size_t syevd_lwork;         // doubles
  const double* pinv_host;    // 32x32 P^-1 block (row-major), host
  const double* pfwd_host;    // 32x32 P block (row-major), host
  const int32_t* perm_host;   // RPBH [K], host
  const float* sgn_host;      // RPBH sign/sqrt(32) [K], host
  double lp = 0.0;             // > 0: robust l_p fit of the residual's block scales
  cudaStream_t stream;
};

// Scratch layout of kq_prepare_weights (float64 throughout).
struct PrepareWs {
  size_t wp = 0, gram = 0, evals = 0, info = 0, work = 0, e = 0, f = 0, sig = 0, l1b = 0,
         l2bt = 0, l1p = 0, pinv = 0, pfwd = 0, total = 0;
  static PrepareWs make(int64_t K, int64_t N, int64_t rank, size_t syevd_lwork);
};

size_t prepare_syevd_lwork(int64_t K, int64_t N, int64_t rank);
PrepStatus run_prepare(const PrepareArgs& a);

}  // namespace kq
