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
// (grouped order, see tile_coords). Warp roles:
//   warp 0     TMA producer: codes tiles (128-byte swizzle) and scale runs (plain bulk
//              copies) into a kStages-deep ring; then the U / L2^T tiles of the tile.
//   warp 1     TMEM allocator and single-thread MMA issuer. Two TMEM accumulators
//              (columns 0 and 192) alternate between tiles, so the epilogue of one tile
//              overlaps the MMAs of the next. Per k-tile: 4 block-scaled MMAs (K = 64
//              each); per tile: 2 or 4 fp16 MMAs (rank <= 32 or <= 64) for the low-rank
//              branch; tcgen05.commit frees
//              ring slots / hands over accumulators.
//   warp 6     scale copier: per k-tile, tcgen05.cp of the stage's block scales into
//              that stage's own TMEM scale set, then a commit the MMA issuer waits on
//              (each tcgen05 instruction costs its issuing thread ~50 cycles, so the
//              copies and the MMAs are issued from two threads).
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, + mu[m] s[n], convert, write a
//              128-byte-swizzled staging tile in shared memory, TMA-store it (async).
// A 192-wide tile whose first row sits in the middle of a 128-row scale atom reads its
// B scales two TMEM columns further on. No TMA multicast is used anywhere.
//
// Codebook variant (template F16): the tensor cores have no format for a Lloyd-Max
// codebook (OrbitQuant section 03), so those layers hand the contraction decoded fp16
// operands (the activation as fp16(sigma level), the residual decoded offline) and the
// main loop runs kind::f16 MMAs over 64-element k-tiles; everything else is shared.
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
constexpr uint32_t kColBytes = 4 * kBN * 4;              // per epilogue warp: s[n0 .. n0 + 191]
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + kColBytes + 1024;
constexpr uint32_t kAccStride = kBN;                     // accumulators at columns 0, 192
constexpr uint32_t kSFCol = 2 * kBN;                     // 384: one scale set per stage
constexpr uint32_t kSFSetCols = 24;                      // SFA 8 columns, then SFB 16
static_assert(kSFCol + kStages * kSFSetCols <= 512, "TMEM columns");
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 224;                            // 7 warps (roles below)
static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");
}  // namespace gemm

// Tile order: groups of kGroupM row tiles, and inside a group every column tile for each
// row tile in turn (row tile fastest). A wave of CTAs then covers a few row tiles across all
// columns, so the activation codes of those rows are re-read from L2 rather than DRAM even
// when the output stream is larger than L2; the weight tiles are shared by all groups.
constexpr int kGroupM = 8;
__device__ __forceinline__ void tile_coords(int tile, int MT, int NT, int& mt, int& nt) {
  const int per_group = kGroupM * NT;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int gm = min(kGroupM, MT - g * kGroupM);           // rows in this (maybe last) group
  mt = g * kGroupM + r % gm;
  nt = r / gm;
}

// F16: the main loop contracts fp16 operands (Lloyd-Max activations decoded to fp16 and
// the residual decoded to fp16) with kind::f16 MMAs, 64 elements (128 bytes) per k-tile;
// the scale copier then only relays the stage barriers.
template <bool OUT_BF16, bool F16>
__global__ void __launch_bounds__(gemm::kThreads, 1) k_gemm_mxf4(const __grid_constant__ GemmParams p) {
  using namespace gemm;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* sf_full = empty + kStages;
  uint64_t* acc_full = sf_full + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  uint8_t* stage0 = smem + 1024;
  uint8_t* epi0 = stage0 + kStages * kStageBytes;
  float* col0 = reinterpret_cast<float*>(epi0 + kEpiBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = static_cast<int>(cdiv(p.M, kBM));
  const int NT = static_cast<int>(cdiv(p.N, kBN));
  const int T = MT * NT;
  const int KT = static_cast<int>(cdiv(p.K, F16 ? 64 : kTileK));
  const bool lowrank = p.rank_pad > 0;
  const int steps = KT + (lowrank ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 1);
    }
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
      grid_dep_wait();                     // codes, scales and U come from the preceding grids
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, MT, NT, mt, nt);
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
          if (ks < KT && F16) {
            mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
            tma_load_2d(a, &p.tmap_a, ks * 64, m0, &full[s]);
            tma_load_2d(b, &p.tmap_b, ks * 64, n0, &full[s]);
          } else if (ks < KT) {
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
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kBM + kBN) * p.rank_pad * 2u);
            tma_load_2d(a, &p.tmap_u, 0, m0, &full[s]);
            tma_load_2d(b, &p.tmap_l2, 0, n0, &full[s]);
          }
        }
      }
      if (!ok) drain_ring(full, kStages, it);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // A tcgen05 instruction costs the issuing thread ~50 cycles, so this thread issues
    // only the MMAs and one commit per k-tile (the scale copies come from warp 6) and
    // does no other arithmetic: descriptors are built once and advanced by constant
    // offsets (start address >> 4 sits in the low bits).
    if (lane == 0) {
      const uint32_t st_addr = smem_u32(stage0);
      const uint64_t adesc0 = sdesc_sw128_kmajor(st_addr);
      const uint64_t bdesc0 = sdesc_sw128_kmajor(st_addr + kABytes);
      constexpr uint32_t kStageDesc = kStageBytes >> 4;
      constexpr uint32_t id0 = idesc_mxf4(kBM, kBN, 0, 0), id2 = idesc_mxf4(kBM, kBN, 2, 2);
      constexpr uint32_t idf16 = idesc_f16(kBM, kBN);              // U and L2^T are fp16
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x, ++local) {
        int mt, nt;
        tile_coords(tile, MT, NT, mt, nt);
        const uint32_t shift = ((nt * kBN) % 128) ? 2u : 0u;
        const int buf = local & 1;
        if (local >= 2 &&
            !mbar_wait(&acc_empty[buf], ((local >> 1) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_ACC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf) * kAccStride;
        for (int ks = 0; ks < steps; ++ks) {
          if (!mbar_wait(&sf_full[s], ph, p.err, KQ_DEV_ERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(s) * kStageDesc;
          const uint64_t ad = adesc0 + so, bd = bdesc0 + so;
          if (ks < KT && F16) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idf16, (ks > 0 || kk > 0) ? 1u : 0u);
          } else if (ks < KT) {
            const uint32_t fa = tmem + kSFCol + static_cast<uint32_t>(s) * kSFSetCols;
            const uint32_t fb = fa + 8 + shift;
            const uint32_t acc0 = ks > 0 ? 1u : 0u;
            const int rem = p.K - ks * kTileK;
            if (rem >= kTileK) {
              mma_mxf4(d, ad, bd, id0, fa, fb, acc0);
              mma_mxf4(d, ad + 2, bd + 2, id2, fa | (2u << 30), fb | (2u << 30), 1u);
              mma_mxf4(d, ad + 4, bd + 4, id0, fa + 4, fb + 8, 1u);
              mma_mxf4(d, ad + 6, bd + 6, id2, (fa + 4) | (2u << 30), (fb + 8) | (2u << 30), 1u);
            } else {
              // last, partial k-tile: only the K-steps of 64 that hold data
              const int nkk = static_cast<int>(cdiv(rem, 64));
              mma_mxf4(d, ad, bd, id0, fa, fb, acc0);
              if (nkk > 1) mma_mxf4(d, ad + 2, bd + 2, id2, fa | (2u << 30), fb | (2u << 30), 1u);
              if (nkk > 2) mma_mxf4(d, ad + 4, bd + 4, id0, fa + 4, fb + 8, 1u);
              if (nkk > 3)
                mma_mxf4(d, ad + 6, bd + 6, id2, (fa + 4) | (2u << 30), (fb + 8) | (2u << 30), 1u);
            }
          } else if (p.rank_pad == 32) {
            const uint32_t a_addr = st_addr + static_cast<uint32_t>(s) * kStageBytes;
            const uint64_t ad64 = sdesc_sw64_kmajor(a_addr), bd64 = sdesc_sw64_kmajor(a_addr + kABytes);
            mma_bf16(d, ad64, bd64, idf16, 1u);
            mma_bf16(d, ad64 + 2, bd64 + 2, idf16, 1u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idf16, 1u);
          }
          tc_commit(&empty[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        tc_commit(&acc_full[buf]);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------- scale copier
    // Per k-tile: the block scales of the stage go from shared memory into that stage's
    // own TMEM scale set (SFA atoms k0, k1; SFB row atoms a0, a0+1 for k0, then k1),
    // then a commit tells the MMA issuer they have landed. A stage's set is rewritten
    // only after the producer refilled the stage, i.e. after the MMAs that read it.
    if (lane == 0) {
      const uint64_t sdesc0 = sdesc_plain_rows16(smem_u32(stage0) + kABytes + kBBytes);
      constexpr uint32_t kStageDesc = kStageBytes >> 4;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
        for (int ks = 0; ks < steps; ++ks) {
          if (!mbar_wait(&full[s], ph, p.err, KQ_DEV_ERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (ks < KT && !F16) {
            const uint32_t fa = tmem + kSFCol + static_cast<uint32_t>(s) * kSFSetCols;
            const uint32_t fb = fa + 8;
            const uint64_t sd = sdesc0 + static_cast<uint64_t>(s) * kStageDesc;
            tmem_cp_32x128b_warpx4(fa, sd);
            tmem_cp_32x128b_warpx4(fa + 4, sd + 32);
            tmem_cp_32x128b_warpx4(fb, sd + 64);
            tmem_cp_32x128b_warpx4(fb + 4, sd + 128);
            tmem_cp_32x128b_warpx4(fb + 8, sd + 96);
            tmem_cp_32x128b_warpx4(fb + 12, sd + 160);
          }
          tc_commit(&sf_full[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------- epilogue
    grid_dep_wait();                       // mu comes from the quantize grid
    const int q = warp & 3;                               // TMEM lane quadrant
    uint8_t* stg = epi0 + static_cast<uint32_t>(q) * kEpiBufs * kEpiBuf;
    float* scol = col0 + q * kBN;                          // this warp's copy of the tile's s
    const uint32_t r8 = static_cast<uint32_t>(lane & 7);
    int local = 0;
    uint32_t nstore = 0;
    for (int tile = blockIdx.x; tile < T; tile += gridDim.x, ++local) {
      int mt, nt;
      tile_coords(tile, MT, NT, mt, nt);
      const int m0 = mt * kBM, n0 = nt * kBN;
      const int buf = local & 1;
      const int row = m0 + 32 * q + lane;
      float mu = 0.f;
      if (p.mu != nullptr) {
        // the row's mean and the tile's 192 column sums, fetched while the MMAs run (the
        // previous tile's reads of scol are done: same warp, in order)
        mu = row < p.M ? p.mu[row] : 0.f;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          const int n = n0 + 32 * c + lane;
          scol[32 * c + lane] = n < p.N ? __ldg(p.s + n) : 0.f;
        }
        __syncwarp();
      }
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait(&acc_full[buf], (local >> 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_ACC));
      tc_fence_after();
      const uint32_t tbase = tmem + static_cast<uint32_t>(buf) * kAccStride +
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
          const float4* s4 = reinterpret_cast<const float4*>(scol + 32 * c);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 sv = s4[j];                       // same address in every lane
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
  auto fn = p.f16 ? k_gemm_mxf4<BF16, true> : k_gemm_mxf4<BF16, false>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(gemm::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = cdiv(p.M, gemm::kBM) * cdiv(p.N, gemm::kBN);
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  // programmatic stream serialization: CTAs may start (barrier init, TMEM allocation,
  // descriptor prefetch) while the quantize grids finish; every read of their outputs
  // sits behind griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = gemm::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fn, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, bool out_bf16, int num_sms, cudaStream_t st) {
  return out_bf16 ? launch_gemm_t<true>(p, num_sms, st) : launch_gemm_t<false>(p, num_sms, st);
}

int gemm_tile_n() { return gemm::kBN; }

}  // namespace kq
