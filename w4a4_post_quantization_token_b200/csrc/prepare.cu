// Offline weight preparation (once per layer), in float64 on the GPU:
//   s   = 1^T W                         (CentriQ abstract: rank-1 restore uses the original W)
//   W'  = P^-1 W                        (KroQuant section 01 identity; OrbitQuant section 03
//                                        folds the inverse rotation into the weight offline)
//   W' ~ L1 L2, rank r                  (SVDQuant explainer section 3: SVD of the updated
//                                        weight, top components kept in 16 bits). The top
//                                        singular pairs come from the eigen-decomposition
//                                        of the smaller Gram matrix (cuBLAS + cuSOLVER).
//   L1 = bf16(U_r S^1/2), L2 = bf16(S^1/2 V_r^T)
//   R   = W' - L1 L2 -> float32 -> MXFP4 along K (residual in 4 bits)
//   L1' = P L1 stored as a bf16 hi/lo pair; c1 = 1^T (hi + lo)
#include <cublas_v2.h>
#include <cusolverDn.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <vector>

#include "kq_prepare.cuh"

namespace kq {

// float64 -> bf16 bits, round to nearest even, directly from float64.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  const uint64_t sign = u >> 63;
  const int ex = static_cast<int>((u >> 52) & 0x7FF);
  if (ex == 0) return static_cast<uint16_t>(sign << 15);               // zero / tiny -> +-0
  uint64_t mant = (u & ((1ull << 52) - 1)) | (1ull << 52);             // 53-bit significand
  int e = ex - 1023;                                                    // x = mant * 2^(e-52)
  // keep 8 significant bits: round mant to a multiple of 2^45
  const uint64_t lsb = (mant >> 45) & 1u;
  const uint64_t rem = mant & ((1ull << 45) - 1);
  const uint64_t half = 1ull << 44;
  mant >>= 45;
  if (rem > half || (rem == half && lsb)) ++mant;
  if (mant == (1ull << 8)) { mant >>= 1; ++e; }
  const int be = e + 127;
  if (be <= 0) return static_cast<uint16_t>(sign << 15);               // below bf16 normals
  if (be >= 255) return static_cast<uint16_t>((sign << 15) | 0x7F80u);  // overflow -> inf
  return static_cast<uint16_t>((sign << 15) | (static_cast<uint32_t>(be) << 7) |
                               static_cast<uint32_t>(mant & 0x7Fu));
}
__device__ __forceinline__ double bf16_bits_to_f64(uint16_t h) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(h) << 16));
}

// s[n] = sum_k W[k, n]
__global__ void k_colsum_bf16(const uint16_t* __restrict__ W, int K, int N, float* __restrict__ s) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  double acc = 0.0;
  for (int k = 0; k < K; ++k) acc += bf16_bits_to_f64(W[static_cast<size_t>(k) * N + n]);
  s[n] = static_cast<float>(acc);
}

// W'[k, n] = (P^-1 W)[k, n], one thread per (32-row block, column).
__global__ void k_fold(const uint16_t* __restrict__ W, int K, int N, int kind,
                       const double* __restrict__ pinv, const int32_t* __restrict__ perm,
                       const float* __restrict__ sgn, double* __restrict__ Wp) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (n >= N) return;
  double w[32];
  if (kind == 2) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      w[j] = bf16_bits_to_f64(W[static_cast<size_t>(perm[32 * b + j]) * N + n]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = bf16_bits_to_f64(W[static_cast<size_t>(32 * b + j) * N + n]);
  }
  const double rs = 1.0 / sqrt(32.0);
#pragma unroll 4
  for (int i = 0; i < 32; ++i) {
    double acc = 0.0;
    if (kind == 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) acc = fma(pinv[32 * i + j], w[j], acc);
    } else if (kind == 2) {
      // (H^T w)[i] with H Sylvester: H[j][i] = (-1)^popcount(i & j)
#pragma unroll
      for (int j = 0; j < 32; ++j) acc += (__popc(i & j) & 1) ? -w[j] : w[j];
      acc = acc * rs * (sgn[32 * b + i] < 0.f ? -1.0 : 1.0);
    } else {
      acc = w[i];
    }
    Wp[static_cast<size_t>(32 * b + i) * N + n] = acc;
  }
}

// Gather the top-r eigenvectors (columns d-1, d-2, ...) of a column-major d x d matrix into
// E (d x r, column-major) and sigma_t = sqrt(max(lambda, 0)).
__global__ void k_take_top(const double* __restrict__ V, const double* __restrict__ lam, int d,
                           int r, double* __restrict__ E, double* __restrict__ sig) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (i < d) E[static_cast<size_t>(t) * d + i] = V[static_cast<size_t>(d - 1 - t) * d + i];
  if (i == 0) sig[t] = sqrt(fmax(lam[d - 1 - t], 0.0));
}

// Build the bf16-rounded factors (as fp64 values) from E (side vectors, scaled by sqrt(sigma))
// and F (the other side, divided by sqrt(sigma)).
//   k_side: E is d x r (d = K when K <= N else N), F is (other dim) x r, both column-major.
__global__ void k_round_factors(const double* __restrict__ E, const double* __restrict__ F,
                                const double* __restrict__ sig, int K, int N, int r, int k_is_d,
                                double* __restrict__ L1b, double* __restrict__ L2bT) {
  // L1b: K x r column-major; L2bT: N x r column-major (= L2^T)
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  const double ss = sqrt(sig[t]);
  const bool live = sig[t] > 0.0;
  if (i < K) {
    const double v = k_is_d ? E[static_cast<size_t>(t) * K + i] * ss
                            : (live ? F[static_cast<size_t>(t) * K + i] / ss : 0.0);
    L1b[static_cast<size_t>(t) * K + i] = bf16_bits_to_f64(f64_to_bf16_bits(v));
  }
  if (i < N) {
    const double v = k_is_d ? (live ? F[static_cast<size_t>(t) * N + i] / ss : 0.0)
                            : E[static_cast<size_t>(t) * N + i] * ss;
    L2bT[static_cast<size_t>(t) * N + i] = bf16_bits_to_f64(f64_to_bf16_bits(v));
  }
}

// Residual R (row-major [K, N] fp64) -> float32 -> MXFP4 along K per column n:
// codes [N, K/2] and scales (tensor-core layout). One thread per (n, block).
__global__ void k_encode_residual(const double* __restrict__ R, int K, int N,
                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                  int64_t katoms, double lp) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (n >= N) return;
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = static_cast<float>(R[static_cast<size_t>(32 * b + j) * N + n]);
  uint32_t c[4];
  // plain OCP rule, or the robust l_p scale fit (CentriQ) when lp > 0
  const uint32_t sb = lp > 0.0 ? mx_encode32_lp(v, lp, c) : mx_encode32(v, c);
  *reinterpret_cast<uint4*>(codes + static_cast<size_t>(n) * (K / 2) + 16 * b) =
      make_uint4(c[0], c[1], c[2], c[3]);
  sf[sf_offset(n, b, katoms)] = static_cast<uint8_t>(sb);
}

// L1' = P L1b (fp64) written as bf16 hi/lo rows of l1t [kUCols, K]: row t = hi of column t,
// row 64 + t = lo of column t. One thread per (32-block, t).
__global__ void k_lift_l1(const double* __restrict__ L1b, int K, int r, int kind,
                          const double* __restrict__ pfwd, const int32_t* __restrict__ perm,
                          const float* __restrict__ sgn, uint16_t* __restrict__ l1t,
                          double* __restrict__ L1p) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (b >= K / 32) return;
  double l[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) l[j] = L1b[static_cast<size_t>(t) * K + 32 * b + j];
  const double rs = 1.0 / sqrt(32.0);
  for (int i = 0; i < 32; ++i) {
    double acc = 0.0;
    int dst = 32 * b + i;
    if (kind == 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) acc = fma(pfwd[32 * i + j], l[j], acc);
    } else if (kind == 2) {
      // (P L)[perm[32b + i]] = sum_j (H/sqrt32)[i][j] sign[32b + j] L[32b + j]
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const double x = (sgn[32 * b + j] < 0.f) ? -l[j] : l[j];
        acc += (__popc(i & j) & 1) ? -x : x;
      }
      acc *= rs;
      dst = perm[32 * b + i];
    } else {
      acc = l[i];
    }
    const uint16_t hi = f64_to_bf16_bits(acc);
    const uint16_t lo = f64_to_bf16_bits(acc - bf16_bits_to_f64(hi));
    l1t[static_cast<size_t>(t) * K + dst] = hi;
    l1t[static_cast<size_t>(kRankPad + t) * K + dst] = lo;
    L1p[static_cast<size_t>(t) * K + dst] = bf16_bits_to_f64(hi) + bf16_bits_to_f64(lo);
  }
}

// c1[t] = sum_k L1p[t][k]   (one block per t)
__global__ void k_rowsum_f64(const double* __restrict__ L1p, int K, float* __restrict__ c1) {
  const int t = blockIdx.x;
  double acc = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) acc += L1p[static_cast<size_t>(t) * K + k];
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) c1[t] = static_cast<float>(red[0]);
}

// l2t[n][t] = fp16 of the bf16-rounded L2[t][n] (exact for |L2| in [2^-14, 65504]) for t < r
__global__ void k_store_l2t(const double* __restrict__ L2bT, int N, int r, uint16_t* __restrict__ l2t) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  for (int t = 0; t < r; ++t) {
    const __half h = __double2half(L2bT[static_cast<size_t>(t) * N + n]);
    l2t[static_cast<size_t>(n) * kRankPad + t] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

// ------------------------------------------------------------------------------------
PrepareWs PrepareWs::make(int64_t K, int64_t N, int64_t rank, size_t syevd_lwork) {
  PrepareWs L;
  const int64_t d = K <= N ? K : N;
  const int64_t r = rank;
  size_t o = 256;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.wp = take(static_cast<size_t>(K) * N * 8);
  L.gram = take(r ? static_cast<size_t>(d) * d * 8 : 8);
  L.evals = take(static_cast<size_t>(d) * 8);
  L.info = take(8);
  L.work = take(r ? syevd_lwork * 8 : 8);
  L.e = take(static_cast<size_t>(d) * (r ? r : 1) * 8);
  L.f = take(static_cast<size_t>(K > N ? K : N) * (r ? r : 1) * 8);
  L.sig = take(static_cast<size_t>(r ? r : 1) * 8);
  L.l1b = take(static_cast<size_t>(K) * (r ? r : 1) * 8);
  L.l2bt = take(static_cast<size_t>(N) * (r ? r : 1) * 8);
  L.l1p = take(static_cast<size_t>(K) * (r ? r : 1) * 8);
  L.pinv = take(32 * 32 * 8);
  L.pfwd = take(32 * 32 * 8);
  L.total = o;
  return L;
}

PrepStatus run_prepare(const PrepareArgs& a) {
  const int K = a.K, N = a.N, r = a.rank;
  const WeightsLayout WL = WeightsLayout::make(K, N, r, a.center, a.kind);
  uint8_t* w = static_cast<uint8_t*>(a.weights);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  const PrepareWs PL = PrepareWs::make(K, N, r, a.syevd_lwork);
  cudaStream_t st = a.stream;
  const uint16_t* W = static_cast<const uint16_t*>(a.W);
  double* Wp = reinterpret_cast<double*>(ws + PL.wp);
  double* pinv = reinterpret_cast<double*>(ws + PL.pinv);
  double* pfwd = reinterpret_cast<double*>(ws + PL.pfwd);
  const int32_t* perm = reinterpret_cast<const int32_t*>(w + WL.perm);
  const float* sgn = reinterpret_cast<const float*>(w + WL.sgn);
#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) return PrepStatus::Cuda; } while (0)

  // clear the whole weights buffer: all padding (scale rows/blocks, low-rank columns) is 0
  CK(cudaMemsetAsync(a.weights, 0, WL.total, st));
  if (a.kind == 2) {
    CK(cudaMemcpyAsync(w + WL.perm, a.perm_host, static_cast<size_t>(K) * 4, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(w + WL.sgn, a.sgn_host, static_cast<size_t>(K) * 4, cudaMemcpyHostToDevice, st));
  }
  CK(cudaMemcpyAsync(pinv, a.pinv_host, 32 * 32 * 8, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(pfwd, a.pfwd_host, 32 * 32 * 8, cudaMemcpyHostToDevice, st));

  k_colsum_bf16<<<static_cast<unsigned>(cdiv(N, 256)), 256, 0, st>>>(W, K, N,
                                                                     reinterpret_cast<float*>(w + WL.s));
  CK(cudaGetLastError());
  k_fold<<<dim3(static_cast<unsigned>(cdiv(N, 128)), K / 32), 128, 0, st>>>(W, K, N, a.kind, pinv,
                                                                             perm, sgn, Wp);
  CK(cudaGetLastError());

  if (r > 0) {
    cublasHandle_t hb = nullptr;
    cusolverDnHandle_t hs = nullptr;
    PrepStatus status = PrepStatus::Ok;
    if (cublasCreate(&hb) != CUBLAS_STATUS_SUCCESS) return PrepStatus::Cuda;
    if (cusolverDnCreate(&hs) != CUSOLVER_STATUS_SUCCESS) { cublasDestroy(hb); return PrepStatus::Cuda; }
    cublasSetStream(hb, st);
    cusolverDnSetStream(hs, st);
    const bool k_is_d = K <= N;
    const int d = k_is_d ? K : N;
    double* G = reinterpret_cast<double*>(ws + PL.gram);
    double* lam = reinterpret_cast<double*>(ws + PL.evals);
    int* info = reinterpret_cast<int*>(ws + PL.info);
    double* work = reinterpret_cast<double*>(ws + PL.work);
    double* E = reinterpret_cast<double*>(ws + PL.e);
    double* F = reinterpret_cast<double*>(ws + PL.f);
    double* sig = reinterpret_cast<double*>(ws + PL.sig);
    double* L1b = reinterpret_cast<double*>(ws + PL.l1b);
    double* L2bT = reinterpret_cast<double*>(ws + PL.l2bt);
    double* L1p = reinterpret_cast<double*>(ws + PL.l1p);
    const double one = 1.0, zero = 0.0, minus1 = -1.0;
    // Wp is row-major [K, N] = column-major Wc (N x K, ld N).
    do {
      cublasStatus_t bs;
      if (k_is_d)   // G = Wc^T Wc  (K x K)
        bs = cublasDgemm(hb, CUBLAS_OP_T, CUBLAS_OP_N, K, K, N, &one, Wp, N, Wp, N, &zero, G, K);
      else          // G = Wc Wc^T  (N x N)
        bs = cublasDgemm(hb, CUBLAS_OP_N, CUBLAS_OP_T, N, N, K, &one, Wp, N, Wp, N, &zero, G, N);
      if (bs != CUBLAS_STATUS_SUCCESS) { status = PrepStatus::Cuda; break; }
      if (cusolverDnDsyevd(hs, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d, G, d, lam, work,
                           static_cast<int>(a.syevd_lwork), info) != CUSOLVER_STATUS_SUCCESS) {
        status = PrepStatus::Cuda; break;
      }
      k_take_top<<<dim3(static_cast<unsigned>(cdiv(d, 256)), r), 256, 0, st>>>(G, lam, d, r, E, sig);
      if (cudaGetLastError() != cudaSuccess) { status = PrepStatus::Cuda; break; }
      if (k_is_d)   // F = Wc E  (N x r): W'^T u
        bs = cublasDgemm(hb, CUBLAS_OP_N, CUBLAS_OP_N, N, r, K, &one, Wp, N, E, K, &zero, F, N);
      else          // F = Wc^T E (K x r): W' v
        bs = cublasDgemm(hb, CUBLAS_OP_T, CUBLAS_OP_N, K, r, N, &one, Wp, N, E, N, &zero, F, K);
      if (bs != CUBLAS_STATUS_SUCCESS) { status = PrepStatus::Cuda; break; }
      k_round_factors<<<dim3(static_cast<unsigned>(cdiv(K > N ? K : N, 256)), r), 256, 0, st>>>(
          E, F, sig, K, N, r, k_is_d ? 1 : 0, L1b, L2bT);
      if (cudaGetLastError() != cudaSuccess) { status = PrepStatus::Cuda; break; }
      // Rc = Wc - L2bT L1b^T  (column-major N x K), i.e. R = W' - L1b L2b
      bs = cublasDgemm(hb, CUBLAS_OP_N, CUBLAS_OP_T, N, K, r, &minus1, L2bT, N, L1b, K, &one, Wp, N);
      if (bs != CUBLAS_STATUS_SUCCESS) { status = PrepStatus::Cuda; break; }
      k_lift_l1<<<dim3(static_cast<unsigned>(cdiv(K / 32, 64)), r), 64, 0, st>>>(
          L1b, K, r, a.kind, pfwd, perm, sgn, reinterpret_cast<uint16_t*>(w + WL.l1t), L1p);
      if (cudaGetLastError() != cudaSuccess) { status = PrepStatus::Cuda; break; }
      k_rowsum_f64<<<r, 256, 0, st>>>(L1p, K, reinterpret_cast<float*>(w + WL.c1));
      k_store_l2t<<<static_cast<unsigned>(cdiv(N, 256)), 256, 0, st>>>(L2bT, N, r,
                                                                        reinterpret_cast<uint16_t*>(w + WL.l2t));
      if (cudaGetLastError() != cudaSuccess) { status = PrepStatus::Cuda; break; }
    } while (false);
    if (status == PrepStatus::Ok) {
      if (cudaStreamSynchronize(st) != cudaSuccess) status = PrepStatus::Cuda;
      int hinfo = 0;
      if (status == PrepStatus::Ok &&
          cudaMemcpy(&hinfo, info, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        status = PrepStatus::Cuda;
      if (status == PrepStatus::Ok && hinfo != 0) status = PrepStatus::Solver;
    }
    cusolverDnDestroy(hs);
    cublasDestroy(hb);
    if (status != PrepStatus::Ok) return status;
  }
  k_encode_residual<<<dim3(static_cast<unsigned>(cdiv(N, 128)), K / 32), 128, 0, st>>>(
      Wp, K, N, w + WL.rcodes, w + WL.rsf, sf_katoms(K), a.lp);
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(st));
#undef CK
  return PrepStatus::Ok;
}

size_t prepare_syevd_lwork(int64_t K, int64_t N, int64_t rank) {
  if (rank <= 0) return 1;
  const int d = static_cast<int>(K <= N ? K : N);
  cusolverDnHandle_t hs = nullptr;
  if (cusolverDnCreate(&hs) != CUSOLVER_STATUS_SUCCESS) return 0;
  int lwork = 0;
  const cusolverStatus_t s = cusolverDnDsyevd_bufferSize(hs, CUSOLVER_EIG_MODE_VECTOR,
                                                         CUBLAS_FILL_MODE_LOWER, d, nullptr, d,
                                                         nullptr, &lwork);
  cusolverDnDestroy(hs);
  if (s != CUSOLVER_STATUS_SUCCESS) return 0;
  return static_cast<size_t>(lwork);
}

// diag(gamma) L1' for the LayerNorm front-end; one block per low-rank column t.
__global__ void k_ln_fold(const uint16_t* __restrict__ l1t, const float* __restrict__ gamma,
                          const float* __restrict__ beta, int K, uint16_t* __restrict__ l1gt,
                          float* __restrict__ cg, float* __restrict__ cb) {
  const int t = blockIdx.x;
  double sg = 0.0, sb = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double v = bf16_bits_to_f64(l1t[static_cast<size_t>(t) * K + k]) +
                     bf16_bits_to_f64(l1t[static_cast<size_t>(kRankPad + t) * K + k]);
    const double vg = static_cast<double>(gamma[k]) * v;
    const uint16_t hi = f64_to_bf16_bits(vg);
    const uint16_t lo = f64_to_bf16_bits(vg - bf16_bits_to_f64(hi));
    l1gt[static_cast<size_t>(t) * K + k] = hi;
    l1gt[static_cast<size_t>(kRankPad + t) * K + k] = lo;
    // gamma^T L1' from the stored pair, the values the MMA multiplies x by: m gamma^T L1'
    // then cancels x diag(gamma) L1' up to fp32 accumulation only
    sg += bf16_bits_to_f64(hi) + bf16_bits_to_f64(lo);
    sb += static_cast<double>(beta[k]) * v;
  }
  __shared__ double rg[256], rb[256];
  rg[threadIdx.x] = sg;
  rb[threadIdx.x] = sb;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      rg[threadIdx.x] += rg[threadIdx.x + w];
      rb[threadIdx.x] += rb[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    cg[t] = static_cast<float>(rg[0]);
    cb[t] = static_cast<float>(rb[0]);
  }
}

cudaError_t launch_ln_fold(const uint16_t* l1t, const float* gamma, const float* beta, int K,
                           uint16_t* l1gt, float* cg, float* cb, cudaStream_t st) {
  k_ln_fold<<<kRankPad, 256, 0, st>>>(l1t, gamma, beta, K, l1gt, cg, cb);
  return cudaGetLastError();
}

}  // namespace kq
