// Conversions between the canonical row-major layouts (codes [rows, K/2], scales
// [rows, K/32], low-rank factors) and the internal tensor-core layouts of the
// prepared-weights buffer and the activation workspace.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kq_pack.cuh"

namespace kq {

// canonical scales [rows, K/32] -> tensor-core layout (padding must be zeroed beforehand)
__global__ void k_sf_to_tiled(const uint8_t* __restrict__ canon, int64_t rows, int K,
                              uint8_t* __restrict__ tiled, int64_t katoms) {
  const int nb = K / kBlock;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= rows * nb) return;
  const int64_t r = t / nb;
  const int b = static_cast<int>(t % nb);
  tiled[sf_offset(r, b, katoms)] = canon[t];
}

__global__ void k_sf_from_tiled(const uint8_t* __restrict__ tiled, int64_t rows, int K,
                                int64_t katoms, uint8_t* __restrict__ canon) {
  const int nb = K / kBlock;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= rows * nb) return;
  const int64_t r = t / nb;
  const int b = static_cast<int>(t % nb);
  canon[t] = tiled[sf_offset(r, b, katoms)];
}

// rows x cols bf16 (row-major, ld_src) -> rows x 64 padded (zero beyond cols)
__global__ void k_pad_cols_bf16(const uint16_t* __restrict__ src, int64_t rows, int cols,
                                uint16_t* __restrict__ dst) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= rows * kRankPad) return;
  const int64_t r = t / kRankPad;
  const int j = static_cast<int>(t % kRankPad);
  dst[t] = j < cols ? src[r * cols + j] : static_cast<uint16_t>(0);
}
__global__ void k_unpad_cols_bf16(const uint16_t* __restrict__ src, int64_t rows, int cols,
                                  uint16_t* __restrict__ dst) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= rows * cols) return;
  const int64_t r = t / cols;
  const int j = static_cast<int>(t % cols);
  dst[t] = src[r * kRankPad + j];
}

// L2 [r, N] bf16 -> l2t [N, 64] fp16 (exact for |L2| in [2^-14, 65504])
__global__ void k_l2_to_l2t(const uint16_t* __restrict__ L2, int r, int N, uint16_t* __restrict__ l2t) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(N) * kRankPad) return;
  const int n = static_cast<int>(t / kRankPad);
  const int j = static_cast<int>(t % kRankPad);
  uint16_t out = 0;
  if (j < r) {
    const float v = __uint_as_float(static_cast<uint32_t>(L2[static_cast<int64_t>(j) * N + n]) << 16);
    const __half h = __float2half_rn(v);
    out = *reinterpret_cast<const uint16_t*>(&h);
  }
  l2t[t] = out;
}
// l2t fp16 -> L2 [r, N] bf16
__global__ void k_l2t_to_l2(const uint16_t* __restrict__ l2t, int r, int N, uint16_t* __restrict__ L2) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(r) * N) return;
  const int j = static_cast<int>(t / N);
  const int n = static_cast<int>(t % N);
  const uint16_t hb = l2t[static_cast<int64_t>(n) * kRankPad + j];
  const float v = __half2float(*reinterpret_cast<const __half*>(&hb));
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  L2[t] = *reinterpret_cast<const uint16_t*>(&b);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits_rn(float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// L1' float32 [K, r] -> l1t rows: t = hi, 64 + t = lo (bf16)
__global__ void k_l1p_to_l1t(const float* __restrict__ L1p, int K, int r, uint16_t* __restrict__ l1t) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(K) * kRankPad) return;
  const int k = static_cast<int>(t / kRankPad);
  const int j = static_cast<int>(t % kRankPad);
  uint16_t hi = 0, lo = 0;
  if (j < r) {
    const float v = L1p[static_cast<int64_t>(k) * r + j];
    hi = f32_to_bf16_bits_rn(v);
    lo = f32_to_bf16_bits_rn(v - __uint_as_float(static_cast<uint32_t>(hi) << 16));
  }
  l1t[static_cast<int64_t>(j) * K + k] = hi;
  l1t[static_cast<int64_t>(kRankPad + j) * K + k] = lo;
}

// c1[j] = sum_k (hi + lo)   (fp64 accumulate), one block per j < 64
__global__ void k_c1_from_l1t(const uint16_t* __restrict__ l1t, int K, int r, float* __restrict__ c1) {
  const int j = blockIdx.x;
  double acc = 0.0;
  if (j < r)
    for (int k = threadIdx.x; k < K; k += blockDim.x)
      acc += static_cast<double>(__uint_as_float(static_cast<uint32_t>(l1t[static_cast<int64_t>(j) * K + k]) << 16)) +
             static_cast<double>(__uint_as_float(static_cast<uint32_t>(l1t[static_cast<int64_t>(kRankPad + j) * K + k]) << 16));
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) c1[j] = static_cast<float>(red[0]);
}

// l1t -> L1' float32 [K, r] = hi + lo
__global__ void k_l1t_to_l1p(const uint16_t* __restrict__ l1t, int K, int r, float* __restrict__ L1p) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(K) * r) return;
  const int k = static_cast<int>(t / r);
  const int j = static_cast<int>(t % r);
  const float hi = __uint_as_float(static_cast<uint32_t>(l1t[static_cast<int64_t>(j) * K + k]) << 16);
  const float lo = __uint_as_float(static_cast<uint32_t>(l1t[static_cast<int64_t>(kRankPad + j) * K + k]) << 16);
  L1p[t] = hi + lo;
}

static inline unsigned grid_for(int64_t n, int block) {
  return static_cast<unsigned>((n + block - 1) / block);
}

#define KQ_LAUNCH(kern, n, ...)                                              \
  do {                                                                       \
    const int64_t n_ = (n);                                                  \
    if (n_ > 0) {                                                            \
      kern<<<grid_for(n_, 256), 256, 0, st>>>(__VA_ARGS__);                  \
      const cudaError_t e_ = cudaGetLastError();                             \
      if (e_ != cudaSuccess) return e_;                                      \
    }                                                                        \
  } while (0)

cudaError_t pack_weights(const WeightsLayout& WL, const uint8_t* r_codes, const uint8_t* r_scales,
                         const float* L1p, const uint16_t* L2, const float* s, uint8_t* w,
                         cudaStream_t st) {
  const int K = static_cast<int>(WL.K), N = static_cast<int>(WL.N), r = static_cast<int>(WL.rank);
  cudaError_t e;
  if ((e = cudaMemsetAsync(w + WL.rcodes, 0, WL.perm - WL.rcodes, st)) != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(w + WL.rcodes, r_codes, static_cast<size_t>(N) * (K / 2),
                           cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  KQ_LAUNCH(k_sf_to_tiled, static_cast<int64_t>(N) * (K / kBlock), r_scales, N, K, w + WL.rsf,
            sf_katoms(K));
  if (r > 0) {
    KQ_LAUNCH(k_l2_to_l2t, static_cast<int64_t>(N) * kRankPad, L2, r, N,
              reinterpret_cast<uint16_t*>(w + WL.l2t));
    KQ_LAUNCH(k_l1p_to_l1t, static_cast<int64_t>(K) * kRankPad, L1p, K, r,
              reinterpret_cast<uint16_t*>(w + WL.l1t));
    k_c1_from_l1t<<<kRankPad, 256, 0, st>>>(reinterpret_cast<const uint16_t*>(w + WL.l1t), K, r,
                                            reinterpret_cast<float*>(w + WL.c1));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = cudaMemcpyAsync(w + WL.s, s, static_cast<size_t>(N) * 4, cudaMemcpyDeviceToDevice, st)) !=
      cudaSuccess)
    return e;
  return cudaSuccess;
}

cudaError_t unpack_weights(const WeightsLayout& WL, const uint8_t* w, uint8_t* r_codes,
                           uint8_t* r_scales, float* L1p, uint16_t* L2, float* c1, float* s,
                           cudaStream_t st) {
  const int K = static_cast<int>(WL.K), N = static_cast<int>(WL.N), r = static_cast<int>(WL.rank);
  cudaError_t e;
  if (r_codes && (e = cudaMemcpyAsync(r_codes, w + WL.rcodes, static_cast<size_t>(N) * (K / 2),
                                      cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (r_scales)
    KQ_LAUNCH(k_sf_from_tiled, static_cast<int64_t>(N) * (K / kBlock), w + WL.rsf, N, K,
              sf_katoms(K), r_scales);
  if (r > 0 && L1p)
    KQ_LAUNCH(k_l1t_to_l1p, static_cast<int64_t>(K) * r, reinterpret_cast<const uint16_t*>(w + WL.l1t),
              K, r, L1p);
  if (r > 0 && L2)
    KQ_LAUNCH(k_l2t_to_l2, static_cast<int64_t>(r) * N, reinterpret_cast<const uint16_t*>(w + WL.l2t),
              r, N, L2);
  if (r > 0 && c1 && (e = cudaMemcpyAsync(c1, w + WL.c1, static_cast<size_t>(r) * 4,
                                          cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (s && (e = cudaMemcpyAsync(s, w + WL.s, static_cast<size_t>(N) * 4, cudaMemcpyDeviceToDevice,
                                st)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t pack_act(const ActLayout& AL, int rank, const uint8_t* codes, const uint8_t* scales,
                     const float* mu, const uint16_t* U, uint8_t* act, cudaStream_t st) {
  const int64_t M = AL.M;
  const int K = static_cast<int>(AL.K);
  cudaError_t e;
  if ((e = cudaMemsetAsync(act, 0, AL.total, st)) != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(act + AL.codes, codes, static_cast<size_t>(M) * (AL.lut ? K * 2 : K / 2),
                           cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (AL.lut) {                                           // per-token sigma
    if ((e = cudaMemcpyAsync(act + AL.sig, scales, static_cast<size_t>(M) * 4,
                             cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  } else {
    KQ_LAUNCH(k_sf_to_tiled, M * (K / kBlock), scales, M, K, act + AL.sf, sf_katoms(K));
  }
  if (mu && (e = cudaMemcpyAsync(act + AL.mu, mu, static_cast<size_t>(M) * 4,
                                 cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (rank > 0 && U)
    KQ_LAUNCH(k_pad_cols_bf16, M * kRankPad, U, M, rank, reinterpret_cast<uint16_t*>(act + AL.u));
  return cudaSuccess;
}

cudaError_t unpack_act(const ActLayout& AL, int rank, const uint8_t* act, uint8_t* codes,
                       uint8_t* scales, float* mu, uint16_t* U, cudaStream_t st) {
  const int64_t M = AL.M;
  const int K = static_cast<int>(AL.K);
  cudaError_t e;
  if (codes && (e = cudaMemcpyAsync(codes, act + AL.codes, static_cast<size_t>(M) * (AL.lut ? K * 2 : K / 2),
                                    cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (scales && AL.lut) {
    if ((e = cudaMemcpyAsync(scales, act + AL.sig, static_cast<size_t>(M) * 4,
                             cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  } else if (scales) {
    KQ_LAUNCH(k_sf_from_tiled, M * (K / kBlock), act + AL.sf, M, K, sf_katoms(K), scales);
  }
  if (mu && (e = cudaMemcpyAsync(mu, act + AL.mu, static_cast<size_t>(M) * 4,
                                 cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (rank > 0 && U)
    KQ_LAUNCH(k_unpad_cols_bf16, M * rank, reinterpret_cast<const uint16_t*>(act + AL.u), M, rank, U);
  return cudaSuccess;
}

// MXFP4 residual (internal layout) -> fp16 [N, K]: E2M1 magnitude x 2^(byte - 127), formed
// exactly in float64 and rounded to nearest even fp16. One thread per 32-element block.
__global__ void k_decode_residual_f16(const uint8_t* __restrict__ rcodes, const uint8_t* __restrict__ rsf,
                                      int64_t N, int K, int64_t katoms, uint16_t* __restrict__ out) {
  const int nb = K / kBlock;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= N * nb) return;
  const int64_t n = t / nb;
  const int b = static_cast<int>(t % nb);
  // E2M1 magnitudes of codes 0..7 (OCP MX: exponent bias 1, one mantissa bit)
  constexpr double kMag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double sc = ldexp(1.0, static_cast<int>(rsf[sf_offset(n, b, katoms)]) - 127);
  const uint8_t* c = rcodes + n * (K / 2) + b * 16;
  uint16_t* o = out + n * K + b * kBlock;
  for (int j = 0; j < kBlock; ++j) {
    const uint32_t code = (c[j / 2] >> (4 * (j & 1))) & 15u;
    const double v = (code & 8u) ? -kMag[code & 7u] * sc : kMag[code & 7u] * sc;
    const __half h = __double2half(v);
    o[j] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

cudaError_t decode_residual_f16(const WeightsLayout& WL, uint8_t* w, cudaStream_t st) {
  const int K = static_cast<int>(WL.K);
  KQ_LAUNCH(k_decode_residual_f16, WL.N * (K / kBlock), w + WL.rcodes, w + WL.rsf, WL.N, K,
            sf_katoms(K), reinterpret_cast<uint16_t*>(w + WL.rf16));
  return cudaSuccess;
}

#undef KQ_LAUNCH

}  // namespace kq
