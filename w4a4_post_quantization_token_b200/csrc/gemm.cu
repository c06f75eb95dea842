// Contraction half of the W4A4 linear layer on the 5th-generation tensor cores:
//
//   Y[m, n] = sum_k deq(Xq)[m, k] deq(Rq)[n, k]          (tcgen05 kind::mxf4, block32)
//           + sum_j U[m, j] L2t[n, j]                     (tcgen05 kind::f16, same accumulator)
//           + mu[m] s[n]                                  (fp32 epilogue)
//
// The first term is the 4-bit x 4-bit product the KroQuant commentary (sections 01, 03)
// and the SVDQuant explainer (section 3) describe; the second is the SVDQuant low-rank
// branch fused into the 4-bit kernel (section 3: Nunchaku fuses the low-rank work into
// the 4-bit kernels); the third is CentriQ's rank-1 full-precision mean restore (abstract).
//
// One CTA computes one 128 x BN output tile. Warp roles:
//   warp 0     TMA producer: codes tiles (128-byte swizzle) and scale runs (plain bulk
//              copies) into a kStages-deep ring; then the U / L2^T tiles.
//   warp 1     TMEM allocator and single-thread MMA issuer: per k-tile, tcgen05.cp the
//              scales into TMEM, 4 block-scaled MMAs (K = 64 each); then 4 bf16 MMAs for
//              the low-rank branch; tcgen05.commit frees ring slots and signals the epilogue.
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, add mu[m] s[n], store.
// No TMA multicast is used anywhere.
#include <cuda_bf16.h>

#include "kq_internal.cuh"

namespace kq {

namespace gemm {
constexpr int kStages = 4;
constexpr int kTileM = 128;
constexpr uint32_t kABytes = kTileM * 128;               // 128 rows x 128 bytes
template <int BN> struct Cfg {
  static constexpr uint32_t kBBytes = BN * 128;
  static constexpr uint32_t kSFABytes = 1024;            // 2 atoms (8 scales per row)
  static constexpr uint32_t kSFBBytes = (BN / 128) * 1024;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
  static constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + 1024;
  static constexpr uint32_t kSFACol = BN;                // TMEM column of the A scales
  static constexpr uint32_t kSFBCol = BN + 32;           // TMEM column of the B scales
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
};
}  // namespace gemm

template <int BN, bool OUT_BF16>
__global__ void __launch_bounds__(192, 1) k_gemm_mxf4(const __grid_constant__ GemmParams p) {
  using namespace gemm;
  using C = Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  uint8_t* stage0 = smem + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int n0 = blockIdx.y * BN;
  const int KT = static_cast<int>(cdiv(p.K, kTileK));
  const bool lowrank = p.rank_pad > 0;
  const int steps = KT + (lowrank ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(accf, 1);
    fence_mbar_init();
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_b);
    if (lowrank) { prefetch_tmap(&p.tmap_u); prefetch_tmap(&p.tmap_l2); }
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* sfa_base = p.sfa + static_cast<size_t>(m0 / 128) * p.katoms * 512u;
      for (int it = 0; it < steps; ++it) {
        const int s = it % kStages;
        if (it >= kStages &&
            !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_EMPTY))
          break;
        uint8_t* a = stage0 + s * C::kStageBytes;
        uint8_t* b = a + kABytes;
        if (it < KT) {
          uint8_t* sfa = b + C::kBBytes;
          uint8_t* sfb = sfa + C::kSFABytes;
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          tma_load_2d(a, &p.tmap_a, it * 128, m0, &full[s]);
          tma_load_2d(b, &p.tmap_b, it * 128, n0, &full[s]);
          bulk_load(sfa, sfa_base + static_cast<size_t>(2 * it) * 512u, 1024, &full[s]);
#pragma unroll
          for (int na = 0; na < BN / 128; ++na) {
            const uint8_t* src = p.sfb + static_cast<size_t>(n0 / 128 + na) * p.katoms * 512u +
                                 static_cast<size_t>(2 * it) * 512u;
            bulk_load(sfb + na * 1024, src, 1024, &full[s]);
          }
        } else {
          mbar_arrive_expect_tx(&full[s], kABytes + C::kBBytes);
          tma_load_2d(a, &p.tmap_u, 0, m0, &full[s]);
          tma_load_2d(b, &p.tmap_l2, 0, n0, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t t_sfa = tmem + C::kSFACol;
      const uint32_t t_sfb = tmem + C::kSFBCol;
      bool ok = true;
      for (int it = 0; it < steps && ok; ++it) {
        const int s = it % kStages;
        ok = mbar_wait(&full[s], (it / kStages) & 1, p.err, KQ_DEV_ERR_TIMEOUT_FULL);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(stage0 + s * C::kStageBytes);
        const uint32_t b = a + kABytes;
        if (it < KT) {
          const uint32_t sfa = b + C::kBBytes;
          const uint32_t sfb = sfa + C::kSFABytes;
#pragma unroll
          for (int ka = 0; ka < 2; ++ka) {
            tmem_cp_32x128b_warpx4(t_sfa + 4 * ka, sdesc_plain_rows16(sfa + 512 * ka));
#pragma unroll
            for (int na = 0; na < BN / 128; ++na)
              tmem_cp_32x128b_warpx4(t_sfb + 8 * ka + 4 * na,
                                     sdesc_plain_rows16(sfb + 1024 * na + 512 * ka));
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t ka = kk >> 1, id = 2u * (kk & 1);
            const uint32_t idesc = idesc_mxf4(kTileM, BN, id, id);
            mma_mxf4(tmem, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                     (t_sfa + 4 * ka) | (id << 30), (t_sfb + 8 * ka) | (id << 30),
                     (it > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          constexpr uint32_t idesc = idesc_bf16(kTileM, BN);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                     1u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
  } else {
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    const bool ok = mbar_wait(accf, 0, p.err, KQ_DEV_ERR_TIMEOUT_ACC);
    tc_fence_after();
    if (ok) {
      const float mu = (p.mu != nullptr && row < p.M) ? p.mu[row] : 0.f;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int nc = n0 + 32 * c;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + 32 * c, r);
        tmem_ld_wait();
        if (row >= p.M || nc >= p.N) continue;
        float y[32];
        const int valid = min(32, p.N - nc);     // N % 16 == 0: 16 or 32
        if (p.mu != nullptr) {
          const float4* s4 = reinterpret_cast<const float4*>(p.s + nc);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 sv = (4 * j < valid) ? __ldg(s4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            y[4 * j + 0] = fmaf(mu, sv.x, __uint_as_float(r[4 * j + 0]));
            y[4 * j + 1] = fmaf(mu, sv.y, __uint_as_float(r[4 * j + 1]));
            y[4 * j + 2] = fmaf(mu, sv.z, __uint_as_float(r[4 * j + 2]));
            y[4 * j + 3] = fmaf(mu, sv.w, __uint_as_float(r[4 * j + 3]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(r[j]);
        }
        if (OUT_BF16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) +
                               static_cast<size_t>(row) * p.N + nc;
          if (valid == 32) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
              pk[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int j = 0; j < 4; ++j) d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid) dst[j] = __float2bfloat16_rn(y[j]);
          }
        } else {
          float* dst = reinterpret_cast<float*>(p.y) + static_cast<size_t>(row) * p.N + nc;
          if (valid == 32) {
            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int j = 0; j < 8; ++j) d4[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid) dst[j] = y[j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, bool BF16>
static cudaError_t launch_gemm_t(const GemmParams& p, cudaStream_t st) {
  using C = gemm::Cfg<BN>;
  auto fn = k_gemm_mxf4<BN, BF16>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmemBytes));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(cdiv(p.M, gemm::kTileM)), static_cast<unsigned>(cdiv(p.N, BN)));
  fn<<<grid, 192, C::kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, int bn, bool out_bf16, cudaStream_t st) {
  if (bn == 256) return out_bf16 ? launch_gemm_t<256, true>(p, st) : launch_gemm_t<256, false>(p, st);
  if (bn == 128) return out_bf16 ? launch_gemm_t<128, true>(p, st) : launch_gemm_t<128, false>(p, st);
  return cudaErrorInvalidValue;
}

}  // namespace kq
