// Online half of the W4A4 linear layer: per-token centring, block transform and
// MXFP4 encoding of bf16 activations, plus the low-rank input U on the tensor cores.
//
//  * k_quantize_rows -- groups of R token rows per CTA step, one thread per 32-element
//    block. Rows are staged in shared memory by a TMA tensor load with the 64-byte swizzle
//    (each block is one 64-byte line, its four 16-byte chunks permuted by line), so that
//    one thread per block reads its block without bank conflicts. Centring (CentriQ abstract: centre each token before
//    the rotation) uses an fp32 per-block sum and an fp64 cross-block sum, then
//    x - mu as (x - mu_hi) - mu_lo in fp32. The block transform runs in registers:
//    Kronecker A^T X_m B with A, B as kernel parameters (KroQuant commentary, section 02),
//    or gather + 32-point fast Walsh-Hadamard + sign (OrbitQuant commentary, section 03,
//    RPBH(X) = X P H D). MXFP4 encoding as in encode.cuh (KroQuant section 03).
//  * k_lowrank_u -- U = X L1' - mu c1 (SVDQuant explainer, section 3: the low-rank branch
//    runs on the high-precision input) as a tcgen05 bf16 GEMM: TMA loads 128x64 tiles of
//    X and of [L1'_hi; L1'_lo; 1], the MMA accumulates 128 x 144 in TMEM, the epilogue
//    forms hi + lo - (rowsum / K) c1 and stores bf16.
#include <cuda_bf16.h>

#include "kq_internal.cuh"

namespace kq {

// ----------------------------------------------------------------------------------
// helpers
// ----------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Physical byte offset of logical byte `off` in a buffer written by a TMA load with the
// 64-byte swizzle (16-byte chunk index XOR address bits 7..8); buffer 512-byte aligned.
__device__ __forceinline__ uint32_t swz64(uint32_t off) {
  return off ^ (((off >> 7) & 3u) << 4);
}

// Load block b (32 bf16) of a swizzled row buffer into fp32 registers.
__device__ __forceinline__ void load_block_swz(const uint8_t* row, int b, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t off = static_cast<uint32_t>(b) * 64u + 16u * c;
    const uint4 q = *reinterpret_cast<const uint4*>(row + swz64(off));
    v[8 * c + 0] = bf16_lo(q.x); v[8 * c + 1] = bf16_hi(q.x);
    v[8 * c + 2] = bf16_lo(q.y); v[8 * c + 3] = bf16_hi(q.y);
    v[8 * c + 4] = bf16_lo(q.z); v[8 * c + 5] = bf16_hi(q.z);
    v[8 * c + 6] = bf16_lo(q.w); v[8 * c + 7] = bf16_hi(q.w);
  }
}

// Gather element e of a swizzled row buffer.
__device__ __forceinline__ float load_elem_swz(const uint8_t* row, int e) {
  const uint32_t off = static_cast<uint32_t>(e) * 2u;
  const uint16_t h = *reinterpret_cast<const uint16_t*>(row + swz64(off));
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ float tree_sum32(const float (&v)[32]) {
  float s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = v[2 * i] + v[2 * i + 1];
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) s[i] = s[i] + s[i + w];
  return s[0];
}

__device__ __forceinline__ double warp_sum_f64(double x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// x (A (x) B) for one block: X_m[i][j] = v[8 i + j], out = A^T X_m B.
__device__ __forceinline__ void kron_apply(float (&v)[32], const float* __restrict__ A,
                                           const float* __restrict__ B) {
  float t[32];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int l = 0; l < 8; ++l) {
      float acc = v[8 * i] * B[l];
#pragma unroll
      for (int j = 1; j < 8; ++j) acc = fmaf(v[8 * i + j], B[8 * j + l], acc);
      t[8 * i + l] = acc;
    }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int l = 0; l < 8; ++l) {
      float acc = A[k] * t[l];
#pragma unroll
      for (int i = 1; i < 4; ++i) acc = fmaf(A[4 * i + k], t[8 * i + l], acc);
      v[8 * k + l] = acc;
    }
}

// In-place 32-point Walsh-Hadamard transform in Sylvester order (unnormalised).
__device__ __forceinline__ void fwht32(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

// ----------------------------------------------------------------------------------
// k_quantize_rows
// ----------------------------------------------------------------------------------
// One CTA processes groups of R consecutive token rows; one thread per 32-element block
// (R * K/32 threads). Groups are staged by TMA (64-byte swizzle, one 64-byte line per
// block) into a ring of up to 4 slots; the CTA walks groups blockIdx.x, +gridDim.x, ...
constexpr int kQMaxBufs = 4;

template <int KIND, bool CENTER, bool DEBUG_XT>
__global__ void __launch_bounds__(512, 1) k_quantize_rows(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int nb = p.K / kBlock;
  const int nb_pad = static_cast<int>(p.katoms) * 4;
  const int R = p.rows_per_group;
  const int items = R * nb;
  const uint32_t grp_bytes = static_cast<uint32_t>(items) * 64u;
  const uint32_t buf_bytes = static_cast<uint32_t>(align_up(grp_bytes, 1024));
  // shared memory carve-up
  const int nbufs = p.nbufs;                                                 // <= kQMaxBufs
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);                       // [nbufs]
  float2* mus = reinterpret_cast<float2*>(smem + 64);                       // [R] (hi, lo)
  uint8_t* sst = smem + 64 + 8 * 64;                                        // scale staging
  float* bsum = reinterpret_cast<float*>(smem + 1024 + align_up(static_cast<size_t>(R) * nb_pad, 16));
  uint8_t* tables = smem + p.tables_off;                                    // RPBH tables
  uint8_t* bufs = smem + p.bufs_off;

  const int ngroups = static_cast<int>(cdiv(p.M, R));
  if (tid == 0) {
    for (int b = 0; b < nbufs; ++b) mbar_init(&full[b], 1);
    fence_mbar_init();
    prefetch_tmap(&p.tmap_x);
  }
  if (KIND == 2) {
    // perm as uint16, block b's 32 entries (64 bytes) with 16-byte chunks swizzled like the rows;
    // sign bits: one 32-bit word per block
    uint16_t* pt = reinterpret_cast<uint16_t*>(tables);
    uint32_t* sb = reinterpret_cast<uint32_t*>(tables + static_cast<size_t>(p.K) * 2);
    for (int k = tid; k < p.K; k += blockDim.x) {
      const uint32_t off = static_cast<uint32_t>(k) * 2u;
      pt[swz64(off) / 2] = static_cast<uint16_t>(p.perm[k]);
    }
    for (int b = tid; b < nb; b += blockDim.x) {
      uint32_t w = 0;
      for (int j = 0; j < 32; ++j) w |= (p.sgn[32 * b + j] < 0.f ? 1u : 0u) << j;
      sb[b] = w;
    }
  }
  __syncthreads();

  auto issue = [&](int g, int buf) {
    uint8_t* dst = bufs + static_cast<size_t>(buf) * buf_bytes;
    mbar_arrive_expect_tx(&full[buf], grp_bytes);
    const int l0 = g * items;
    for (int l = 0; l < items; l += p.box_lines)
      tma_load_2d(dst + static_cast<size_t>(l) * 64u, &p.tmap_x, 0, l0 + l, &full[buf]);
  };
  if (tid == 0)
    for (int b = 0; b < nbufs; ++b) {
      const int g = blockIdx.x + b * gridDim.x;
      if (g < ngroups) issue(g, b);
    }

  int iter = 0;
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x, ++iter) {
    const int buf = iter % nbufs;
    const uint32_t parity = static_cast<uint32_t>(iter / nbufs) & 1u;
    const int row0 = g * R;
    __syncthreads();   // previous group's staging reads are done
    const bool ok = __syncthreads_and(mbar_wait(&full[buf], parity, p.err, KQ_DEV_ERR_TIMEOUT_FULL));
    if (!ok) break;
    const uint8_t* gbuf = bufs + static_cast<size_t>(buf) * buf_bytes;

    if (CENTER) {
      for (int i = tid; i < items; i += blockDim.x) {
        float v[32];
        load_block_swz(gbuf, i, v);
        bsum[i] = tree_sum32(v);
      }
      __syncthreads();
      const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
      for (int r = warp; r < R; r += nwarps) {
        double part = 0.0;
        for (int b = lane; b < nb; b += 32) part += static_cast<double>(bsum[r * nb + b]);
        const double mu64 = warp_sum_f64(part) / static_cast<double>(p.K);
        const float hi = static_cast<float>(mu64);
        const float lo = static_cast<float>(mu64 - static_cast<double>(hi));
        if (lane == 0) {
          mus[r] = make_float2(hi, lo);
          if (row0 + r < p.M) p.mu[row0 + r] = hi;
        }
      }
      __syncthreads();
    } else if (tid < R && row0 + tid < p.M) {
      p.mu[row0 + tid] = 0.f;
    }

    for (int i = tid; i < items; i += blockDim.x) {
      const int r = i / nb, b = i - r * nb;
      const int row = row0 + r;
      if (row >= p.M) continue;
      float v[32];
      // swizzle positions are taken relative to the 1024-byte aligned ring slot: line index
      // i = r * nb + b for the block, element index r * K + e for a gathered element
      if (KIND == 2) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 ix = *reinterpret_cast<const uint4*>(
              tables + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
          const uint32_t w4[4] = {ix.x, ix.y, ix.z, ix.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            v[8 * c + 2 * t] = load_elem_swz(gbuf, r * p.K + static_cast<int>(w4[t] & 0xFFFFu));
            v[8 * c + 2 * t + 1] = load_elem_swz(gbuf, r * p.K + static_cast<int>(w4[t] >> 16));
          }
        }
      } else {
        load_block_swz(gbuf, i, v);
      }
      if (CENTER) {
        const float2 m = mus[r];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (v[j] - m.x) - m.y;
      }
      if (KIND == 1) {
        kron_apply(v, p.A, p.B);
      } else if (KIND == 2) {
        fwht32(v);
        const uint32_t sbits = reinterpret_cast<const uint32_t*>(tables + static_cast<size_t>(p.K) * 2)[b];
        const float rs = 0.17677669529663687f;   // 1 / sqrt(32)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = __uint_as_float(__float_as_uint(v[j] * rs) ^ (((sbits >> j) & 1u) << 31));
      }
      if (DEBUG_XT) {
        float4* o = reinterpret_cast<float4*>(p.xt + static_cast<size_t>(row) * p.K + b * kBlock);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        uint32_t c[4];
        const uint32_t sbyte = mx_encode32(v, c);
        *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * (p.K / 2) + b * 16) =
            make_uint4(c[0], c[1], c[2], c[3]);
        sst[r * nb_pad + b] = static_cast<uint8_t>(sbyte);
      }
    }
    __syncthreads();   // all reads of this ring slot and all staged scales are done
    if (tid == 0) {
      const int gn = g + nbufs * gridDim.x;
      if (gn < ngroups) {
        fence_async_smem();
        issue(gn, buf);
      }
    }
    if (!DEBUG_XT) {
      // scale words: 4 consecutive blocks of one row per 32-bit word, padding blocks = 0
      const int wpr = nb_pad / 4;
      for (int i = tid; i < R * wpr; i += blockDim.x) {
        const int r = i / wpr, w = i - r * wpr;
        const int row = row0 + r;
        if (row >= p.M) continue;
        uint32_t word = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int b = 4 * w + t;
          const uint32_t v = b < nb ? sst[r * nb_pad + b] : 0u;
          word |= v << (8 * t);
        }
        *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, 4 * w, p.katoms)) = word;
      }
    }
  }
  // rows M .. m_pad-1 of the last 128-row group: zero scales (finite values for the GEMM)
  if (!DEBUG_XT) {
    const int wpr = nb_pad / 4;
    const int pad_rows = p.m_pad - p.M;
    for (int i = blockIdx.x * blockDim.x + tid; i < pad_rows * wpr; i += gridDim.x * blockDim.x) {
      const int r = p.M + i / wpr, w = i % wpr;
      *reinterpret_cast<uint32_t*>(p.sf + sf_offset(r, 4 * w, p.katoms)) = 0u;
      if (w == 0) p.mu[r] = 0.f;
    }
  }
}

// ----------------------------------------------------------------------------------
// k_encode_f32 (debug): encoder alone on float32 rows, canonical outputs
// ----------------------------------------------------------------------------------
__global__ void k_encode_f32(const float* __restrict__ V, int M, int K, uint8_t* __restrict__ codes,
                             uint8_t* __restrict__ scales) {
  const int nb = K / kBlock;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(M) * nb) return;
  const int64_t row = t / nb;
  const int b = static_cast<int>(t % nb);
  const float4* src = reinterpret_cast<const float4*>(V + row * K + b * kBlock);
  float v[32];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 f = src[q];
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
  uint32_t c[4];
  const uint32_t sb = mx_encode32(v, c);
  *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = make_uint4(c[0], c[1], c[2], c[3]);
  scales[row * nb + b] = static_cast<uint8_t>(sb);
}

// ----------------------------------------------------------------------------------
// k_lowrank_u: U[m, 0..63] = X L1'_hi + X L1'_lo - (center ? rowsum/K : 0) * c1
// ----------------------------------------------------------------------------------
namespace lowrank {
constexpr int kStages = 4;
constexpr int kTileM = 128;
constexpr int kChunkK = 64;                      // bf16 elements per stage (128 bytes)
constexpr uint32_t kABytes = kTileM * 128;       // 16 KB
constexpr uint32_t kBBytes = kUCols * 128;       // 18 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + 1024;
constexpr uint32_t kTmemCols = 256;
}  // namespace lowrank

__global__ void __launch_bounds__(192, 1) k_lowrank_u(const __grid_constant__ LowRankParams p) {
  using namespace lowrank;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  uint8_t* stage0 = smem + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int KT = static_cast<int>(cdiv(p.K, kChunkK));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(accf, 1);
    fence_mbar_init();
    prefetch_tmap(&p.tmap_x);
    prefetch_tmap(&p.tmap_l1);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (kt >= kStages &&
            !mbar_wait(&empty[s], ((kt / kStages) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_EMPTY))
          break;
        uint8_t* a = stage0 + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(a, &p.tmap_x, kt * kChunkK, m0, &full[s]);
        tma_load_2d(a + kABytes, &p.tmap_l1, kt * kChunkK, 0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTileM, kUCols);
      bool ok = true;
      for (int kt = 0; kt < KT && ok; ++kt) {
        const int s = kt % kStages;
        ok = mbar_wait(&full[s], (kt / kStages) & 1, p.err, KQ_DEV_ERR_TIMEOUT_FULL);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(stage0 + s * kStageBytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int kk = 0; kk < kChunkK / 16; ++kk)
          mma_bf16(tmem, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                   (kt > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
  } else {
    // epilogue warps 2..5: TMEM lane quadrant = warp % 4
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    const bool ok = mbar_wait(accf, 0, p.err, KQ_DEV_ERR_TIMEOUT_ACC);
    tc_fence_after();
    if (ok) {
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16);
      uint32_t hi0[32], hi1[32], lo0[32], lo1[32], sm[32];
      tmem_ld_32x32b_x32(tbase + 0, hi0);
      tmem_ld_32x32b_x32(tbase + 32, hi1);
      tmem_ld_32x32b_x32(tbase + 64, lo0);
      tmem_ld_32x32b_x32(tbase + 96, lo1);
      tmem_ld_32x32b_x32(tbase + 128, sm);
      tmem_ld_wait();
      const float mu = p.center ? __uint_as_float(sm[0]) / static_cast<float>(p.K) : 0.f;
      if (row < p.M) {
        uint32_t packed[32];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float a0 = __uint_as_float(hi0[j]) + __uint_as_float(lo0[j]) - mu * p.c1[j];
          const float a1 = __uint_as_float(hi0[j + 1]) + __uint_as_float(lo0[j + 1]) - mu * p.c1[j + 1];
          const float b0 = __uint_as_float(hi1[j]) + __uint_as_float(lo1[j]) - mu * p.c1[32 + j];
          const float b1 = __uint_as_float(hi1[j + 1]) + __uint_as_float(lo1[j + 1]) - mu * p.c1[33 + j];
          const __nv_bfloat162 pa = __floats2bfloat162_rn(a0, a1);
          const __nv_bfloat162 pb = __floats2bfloat162_rn(b0, b1);
          packed[j / 2] = *reinterpret_cast<const uint32_t*>(&pa);
          packed[16 + j / 2] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        uint4* dst = reinterpret_cast<uint4*>(p.u + static_cast<size_t>(row) * kRankPad);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------------
template <int KIND, bool CENTER, bool DBG>
static cudaError_t launch_rows_t(const QuantParams& p, int num_sms, int block, size_t smem,
                                 cudaStream_t st) {
  auto fn = k_quantize_rows<KIND, CENTER, DBG>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, block, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int64_t groups = cdiv(p.M, p.rows_per_group);
  int64_t grid = static_cast<int64_t>(num_sms) * per_sm;
  if (grid > groups) grid = groups;
  if (grid < 1) grid = 1;
  fn<<<static_cast<unsigned>(grid), block, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const QuantParams& p, bool debug_xt, int num_sms,
                                 cudaStream_t st) {
  const int items = p.rows_per_group * (p.K / kBlock);
  int block = static_cast<int>(align_up(static_cast<size_t>(items), 32));
  if (block > 512) block = 512;
  const size_t smem = p.smem_bytes;
  const int kind = p.kind, c = p.center ? 1 : 0;
#define KQ_DISPATCH(KD, C)                                                             \
  if (kind == KD && c == C)                                                            \
    return debug_xt ? launch_rows_t<KD, (C != 0), true>(p, num_sms, block, smem, st)   \
                    : launch_rows_t<KD, (C != 0), false>(p, num_sms, block, smem, st);
  KQ_DISPATCH(0, 0) KQ_DISPATCH(0, 1) KQ_DISPATCH(1, 0) KQ_DISPATCH(1, 1) KQ_DISPATCH(2, 0)
  KQ_DISPATCH(2, 1)
#undef KQ_DISPATCH
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode_f32(const float* V, int M, int K, uint8_t* codes, uint8_t* scales,
                              cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(M) * (K / kBlock);
  const int block = 256;
  const int64_t grid = cdiv(n, block);
  if (n == 0) return cudaSuccess;
  k_encode_f32<<<static_cast<unsigned>(grid), block, 0, st>>>(V, M, K, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_lowrank_u(const LowRankParams& p, cudaStream_t st) {
  using namespace lowrank;
  cudaError_t e = cudaFuncSetAttribute(k_lowrank_u, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t grid = cdiv(p.M, kTileM);
  k_lowrank_u<<<static_cast<unsigned>(grid), 192, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace kq
