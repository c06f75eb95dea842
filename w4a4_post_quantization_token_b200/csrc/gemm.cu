// Contraction half of the W4A4 linear layer on the 5th-generation tensor cores:
//
//   Y[m, n] = sum_k deq(Xq)[m, k] deq(Rq)[n, k]          (tcgen05 kind::mxf4, block32)
//           + sum_j U[m, j] L2t[n, j]                     (tcgen05 kind::f16, fp16, same accumulator)
//           + mu[m] s[n]                                  (fp32 epilogue)
//
// The first term is the 4-bit x 4-bit product the KroQuant commentary (sections 01, 03)
// and the SVDQuant explainer (section 3) describe; the second is the SVDQuant low-rank
// branch fused into the 4-bit kernel (section 3: Nunchaku fuses the low-rank work into
// the 4-bit kernels); the third is CentriQ's rank-1 full-precision mean restore (abstract).
//
// Persistent kernel, one CTA per SM, static round-robin over 128 x 192 output tiles
// (M fastest). Warp roles:
//   warp 0     TMA producer: codes tiles (128-byte swizzle) and scale runs (plain bulk
//              copies) into a kStages-deep ring; then the U / L2^T tiles of the tile.
//   warp 1     TMEM allocator and single-thread MMA issuer. Two TMEM accumulators
//              (2 x 192 columns) alternate between tiles, so the epilogue of one tile
//              overlaps the MMAs of the next. Per k-tile: tcgen05.cp of the scales into
//              TMEM, then block-scaled MMAs (K = 64 each); per tile: 4 fp16 MMAs for the
//              low-rank branch; tcgen05.commit frees ring slots / hands over accumulators.
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, + mu[m] s[n], convert, write a
//              128-byte-swizzled staging tile in shared memory, TMA-store it (async).
// A 192-wide tile whose first row sits in the middle of a 128-row scale atom reads its
// B scales two TMEM columns further on. No TMA multicast is used anywhere.
#include <cuda_bf16.h>

#include "kq_internal.cuh"

namespace kq {

namespace gemm {
constexpr int kStages = 4;
constexpr int kBM = 128;
constexpr int kBN = 192;
constexpr uint32_t kABytes = kBM * 128;                  // 128 rows x 128 bytes
constexpr uint32_t kBBytes = kBN * 128;                  // 192 rows x 128 bytes
constexpr uint32_t kSFABytes = 1024;                     // 2 atoms (8 scales per row)
constexpr uint32_t kSFBBytes = 2048;                     // 2 row atoms x 2 k atoms
constexpr uint32_t kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
constexpr uint32_t kEpiBuf = 4096;                       // 32 rows x 128 bytes
constexpr int kEpiBufs = 2;                              // per epilogue warp
constexpr uint32_t kEpiBytes = 4 * kEpiBufs * kEpiBuf;
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + 1024;
constexpr uint32_t kAccCols = kBN;                       // one accumulator
constexpr uint32_t kSFACol = 2 * kBN;                    // 384
constexpr uint32_t kSFBCol = 2 * kBN + 32;               // 416
constexpr uint32_t kTmemCols = 512;
static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");
}  // namespace gemm

template <bool OUT_BF16>
__global__ void __launch_bounds__(192, 1) k_gemm_mxf4(const __grid_constant__ GemmParams p) {
  using namespace gemm;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  uint8_t* stage0 = smem + 1024;
  uint8_t* epi0 = stage0 + kStages * kStageBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = static_cast<int>(cdiv(p.M, kBM));
  const int NT = static_cast<int>(cdiv(p.N, kBN));
  const int T = MT * NT;
  const int KT = static_cast<int>(cdiv(p.K, kTileK));
  const bool lowrank = p.rank_pad > 0;
  const int steps = KT + (lowrank ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 4); }
    fence_mbar_init();
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_b);
    prefetch_tmap(&p.tmap_y);
    if (lowrank) { prefetch_tmap(&p.tmap_u); prefetch_tmap(&p.tmap_l2); }
  }
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
        const int mt = tile % MT, nt = tile / MT;
        const int m0 = mt * kBM, n0 = nt * kBN;
        const int a0 = n0 / 128;
        const uint8_t* sfa_base = p.sfa + static_cast<size_t>(mt) * p.katoms * 512u;
        const uint8_t* sfb_base0 = p.sfb + static_cast<size_t>(a0) * p.katoms * 512u;
        const uint8_t* sfb_base1 = sfb_base0 + static_cast<size_t>(p.katoms) * 512u;
        for (int ks = 0; ks < steps; ++ks, ++it) {
          const int s = it % kStages;
          if (it >= kStages &&
              !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* a = stage0 + s * kStageBytes;
          uint8_t* b = a + kABytes;
          if (ks < KT) {
            uint8_t* sfa = b + kBBytes;
            uint8_t* sfb = sfa + kSFABytes;
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_2d(a, &p.tmap_a, ks * 128, m0, &full[s]);
            tma_load_2d(b, &p.tmap_b, ks * 128, n0, &full[s]);
            const size_t ko = static_cast<size_t>(2 * ks) * 512u;
            bulk_load(sfa, sfa_base + ko, 1024, &full[s]);
            bulk_load(sfb, sfb_base0 + ko, 1024, &full[s]);
            bulk_load(sfb + 1024, sfb_base1 + ko, 1024, &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
            tma_load_2d(a, &p.tmap_u, 0, m0, &full[s]);
            tma_load_2d(b, &p.tmap_l2, 0, n0, &full[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t t_sfa = tmem + kSFACol;
      const uint32_t t_sfb = tmem + kSFBCol;
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x, ++local) {
        const int nt = tile / MT;
        const int n0 = nt * kBN;
        const uint32_t shift = (n0 % 128) ? 2u : 0u;
        const int buf = local & 1;
        if (local >= 2 &&
            !mbar_wait(&acc_empty[buf], ((local >> 1) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_ACC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf) * kAccCols;
        for (int ks = 0; ks < steps; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], (it / kStages) & 1, p.err, KQ_DEV_ERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(stage0 + s * kStageBytes);
          const uint32_t b = a + kABytes;
          if (ks < KT) {
            const uint32_t sfa = b + kBBytes;
            const uint32_t sfb = sfa + kSFABytes;
#pragma unroll
            for (int ka = 0; ka < 2; ++ka) {
              tmem_cp_32x128b_warpx4(t_sfa + 4 * ka, sdesc_plain_rows16(sfa + 512 * ka));
              tmem_cp_32x128b_warpx4(t_sfb + 8 * ka, sdesc_plain_rows16(sfb + 512 * ka));
              tmem_cp_32x128b_warpx4(t_sfb + 8 * ka + 4, sdesc_plain_rows16(sfb + 1024 + 512 * ka));
            }
            // K-steps of 64 elements that hold data (the last k-tile may be a partial one)
            const int rem = p.K - ks * kTileK;
            const int nkk = rem >= kTileK ? 4 : static_cast<int>(cdiv(rem, 64));
            for (int kk = 0; kk < nkk; ++kk) {
              const uint32_t ka = kk >> 1, id = 2u * (kk & 1);
              const uint32_t idesc = idesc_mxf4(kBM, kBN, id, id);
              mma_mxf4(d, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                       (t_sfa + 4 * ka) | (id << 30), (t_sfb + 8 * ka + shift) | (id << 30),
                       (ks > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
            constexpr uint32_t idesc = idesc_f16(kBM, kBN);      // U and L2^T are fp16
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                       1u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;                               // TMEM lane quadrant
    uint8_t* stg = epi0 + static_cast<uint32_t>(q) * kEpiBufs * kEpiBuf;
    const uint32_t r8 = static_cast<uint32_t>(lane & 7);
    int local = 0;
    uint32_t nstore = 0;
    for (int tile = blockIdx.x; tile < T; tile += gridDim.x, ++local) {
      const int mt = tile % MT, nt = tile / MT;
      const int m0 = mt * kBM, n0 = nt * kBN;
      const int buf = local & 1;
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait(&acc_full[buf], (local >> 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_ACC));
      tc_fence_after();
      const int row = m0 + 32 * q + lane;
      const float mu = (p.mu != nullptr && row < p.M) ? p.mu[row] : 0.f;
      const uint32_t tbase = tmem + static_cast<uint32_t>(buf) * kAccCols +
                             (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + 32 * c, r);
        tmem_ld_wait();
        if (c == kBN / 32 - 1) {
          // every column of this accumulator is in registers: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        if (!ok) continue;
        const int nc = n0 + 32 * c;
        float y[32];
        if (p.mu != nullptr) {
          const int valid = min(32, p.N - nc);
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
        // staging: 32 rows x 128 bytes, 16-byte chunk j of row r stored at chunk j ^ (r % 8)
        const bool first_half = OUT_BF16 ? ((c & 1) == 0) : true;
        const bool last_half = OUT_BF16 ? ((c & 1) == 1) : true;
        uint8_t* sb = stg + (nstore % kEpiBufs) * kEpiBuf;
        if (first_half) {
          if (lane == 0) bulk_wait_read<kEpiBufs - 1>();
          __syncwarp();
        }
        uint8_t* rowp = sb + static_cast<uint32_t>(lane) * 128u;
        if (OUT_BF16) {
          const uint32_t h = static_cast<uint32_t>(c & 1);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t pk[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(y[8 * j + 2 * t], y[8 * j + 2 * t + 1]);
              pk[t] = *reinterpret_cast<const uint32_t*>(&v2);
            }
            const uint32_t chunk = (4u * h + j) ^ r8;
            *reinterpret_cast<uint4*>(rowp + 16u * chunk) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t chunk = static_cast<uint32_t>(j) ^ r8;
            *reinterpret_cast<float4*>(rowp + 16u * chunk) =
                make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
          }
        }
        if (last_half) {
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int x = OUT_BF16 ? n0 + 64 * (c >> 1) : nc;
            tma_store_2d(&p.tmap_y, sb, x, m0 + 32 * q);
            bulk_commit();
          }
          ++nstore;
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool BF16>
static cudaError_t launch_gemm_t(const GemmParams& p, int num_sms, cudaStream_t st) {
  auto fn = k_gemm_mxf4<BF16>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(gemm::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = cdiv(p.M, gemm::kBM) * cdiv(p.N, gemm::kBN);
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  fn<<<grid, 192, gemm::kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, bool out_bf16, int num_sms, cudaStream_t st) {
  return out_bf16 ? launch_gemm_t<true>(p, num_sms, st) : launch_gemm_t<false>(p, num_sms, st);
}

int gemm_tile_n() { return gemm::kBN; }

}  // namespace kq
