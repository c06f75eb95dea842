// Internal declarations shared by the library's translation units: kernel parameter
// blocks and launcher prototypes.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "encode.cuh"
#include "layout.cuh"
#include "sm100.cuh"

namespace kq {

constexpr int kQMaxWarps = 16;        // warps per quantize CTA
constexpr int kQMaxWarpsKron = 16;    // Kronecker (FMA-bound): as many warps as fit
constexpr int kQMaxStages = 3;        // slots per consumer warp
constexpr int kQMuOff = 1024;         // smem offset of the per-warp token means
constexpr int kQTablesMin = kQMuOff + kQMaxWarps * 32 * 8;
// LayerNorm front-end: per-row float4 (rstd, mean_y hi, mean_y lo, 0) after the means
constexpr int kQLnOff = kQTablesMin;
constexpr int kQTablesMinLn = kQLnOff + kQMaxWarps * 32 * 16;
// dynamic shared memory of one k_lowrank_u CTA (3 stages of 32 KB + barriers)
constexpr size_t kLowRankSmemBytes = 1024 + 3 * 32768 + 1024;
constexpr size_t kSmemPerSM = 233472;          // B200: 228 KB per SM
constexpr size_t kSmemPerBlockReserved = 1024; // taken by the driver for every resident CTA

struct QuantParams {
  CUtensorMap tmap_x;          // X viewed as [M * K/32 lines, 32 bf16], 64-byte swizzle
  uint64_t Ap[16];             // Kronecker A as pairs (A[i][k], A[i][k]), index 4 i + k
  uint64_t Bp[32];             // Kronecker B as pairs (B[j][2l], B[j][2l+1]), index 4 j + l
  int M, K, m_pad, center;
  int kind;                    // 0 none, 1 Kronecker, 2 RPBH, 3 per-channel scale
  int unit_rows;               // rows per work unit (one consumer warp at a time)
  int consumer_warps;          // warps per CTA, <= kQMaxWarps (kQMaxWarpsKron)
  int box_lines;               // 64-byte lines per TMA box (divides K/32, <= 256)
  int nbufs;                   // slots per consumer warp (<= kQMaxStages)
  uint32_t row_stride;         // bytes between staged rows (512-byte multiple)
  uint32_t qtab_bytes;         // RPBH table bytes (K * 2 + K/32 * 16)
  size_t tables_off, bufs_off, smem_bytes;   // dynamic shared memory carve-up
  int64_t katoms;
  uint8_t* codes;              // act codes [M, K/2]
  uint8_t* sf;                 // act scales (tensor-core layout)
  float* mu;                   // [m_pad]
  const uint8_t* qtab;         // RPBH shared-memory table image (weights buffer)
  const float* inv_s;          // kind 3 (SmoothQuant comparator): fp32 [K] inverse channel scales
  int ln;                      // LayerNorm front-end on (needs center)
  double ln_eps;
  const uint8_t* lntab;        // LayerNorm table image (weights buffer), ln_table_bytes
  uint32_t lntab_bytes;
  uint32_t lntab_off;          // its shared-memory offset (128-byte aligned)
  float* lnm;                  // out: per-token mean of x [m_pad]
  float* lnr;                  // out: per-token 1/sqrt(v + eps) [m_pad]
  int keep_err;                // 1: leave the device error word as it is (later row chunks
                               //    of one call), 0: clear it first
  int lut;                     // Lloyd-Max activations: fp16 operand out, no block scales
  float lut_mag[8];            //   positive codebook levels (ascending)
  float lut_thr[7];            //   thresholds between them
  uint16_t* a16;               // out: fp16 operand [M, K]
  float* sig;                  // out: per-token sigma [m_pad]
  float* xt;                   // debug: transformed values [M, K] (debug launch only)
  uint32_t* err;
};

struct LowRankParams {
  CUtensorMap tmap_x;          // X [M, K] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap tmap_l1;         // [kUCols, K] bf16, box 64 x kUCols, 128-byte swizzle
  int lowrank;                 // 1: U = X L1' - mu c1 (rank > 0); 0: statistics only
  int stats;                   // 1: form the token means from the streamed X (centring) and
                               //    write them; 0: read them from `mu` (or none)
  int clear_err;               // first kernel of the call: clear the device error word
  int m_pad;                   // rows of the padded workspace (mu_out is zeroed up to it)
  float* mu_out;               // stats: fp32(mu) [m_pad]
  float* mulo_out;             // stats: fp32(mu - fp32(mu)) for rows < M, at row * mulo_stride
  int64_t mulo_stride;
  const float* c1;             // [64]
  const float* mu;             // [M] token means (null without centring, unused with stats)
  uint16_t* u;                 // U [M, 64] fp16
  int deep;                    // 1: the quantize CTAs leave no room on the SM, use the deep ring
  int reverse;                 // 1: take the row tiles from the last to the first (after k_quantize_rows)
  int ln;                      // LayerNorm front-end: L1 map is diag(gamma) L1', and
  const float* cg;             //   U = rstd acc - rstd m cg + cb - mu c1 with cg = gamma^T L1'
  const float* cb;             //   and cb = beta^T L1' [64]
  const float* lnm;            //   per-token m and rstd from the quantize kernel
  const float* lnr;
  int M, K, split;             // split: CTAs (one cluster) per 128-row tile, 1/2/4/8
  uint32_t* err;
};

// k_quantize_chunks: the online half for the Kronecker transform (or none) on 128-row x
// 64-element pieces of X, with the token means already formed by k_lowrank_u (stats).
struct ChunkParams {
  CUtensorMap tmap_x;          // X [M, K] bf16, box 64 x 128, 128-byte swizzle
  uint64_t Ap[16];             // Kronecker A as pairs (A[i][k], A[i][k]), index 4 i + k
  uint64_t Bp[32];             // Kronecker B as pairs (B[j][2l], B[j][2l+1]), index 4 j + l
  float colsumA[4];            // Kronecker: sum_i A[i][k] and sum_j B[j][l] (1^T P = sA (x) sB)
  float colsumB[8];
  int M, K, m_pad;
  int tiles;                   // cdiv(M, 128)
  int pairs;                   // pieces of 4 blocks per row: cdiv(K, 128)
  int clear_err;               // first kernel of the call: clear the device error word
  int64_t katoms;
  const float* mu;             // centring: fp32(mu) [M]
  const float* mulo;           // centring: fp32(mu - fp32(mu)), row r at r * mulo_stride
  int64_t mulo_stride;
  float* mu_clear;             // no centring: the workspace's means [m_pad], set to 0 here
  uint8_t* codes;              // act codes [M, K/2]
  uint8_t* sf;                 // act scales (tensor-core layout, rows padded to m_pad)
  float* xt;                   // debug: transformed values [M, K] instead of codes / scales
  uint32_t* err;
};

struct GemmParams {
  CUtensorMap tmap_a;          // act codes [M, K/2] uint8, box 128 x 128, 128-byte swizzle
  CUtensorMap tmap_b;          // residual codes [N, K/2] uint8, box 128 x BN
  CUtensorMap tmap_u;          // U [M, 64] fp16, box rank_pad x 128
  CUtensorMap tmap_l2;         // L2^T [N, 64] fp16, box rank_pad x BN
  CUtensorMap tmap_y;          // Y [M, N] f32 or bf16, box (128 bytes) x 32 rows, 128-byte swizzle
  const uint8_t* sfa;          // act scales (tensor-core layout)
  const uint8_t* sfb;          // residual scales (tensor-core layout, one spare row atom)
  const float* mu;             // [M] or null (no centring)
  const float* s;              // [N]
  void* y;                     // [M, N] f32 or bf16
  int M, N, K;
  int rank_pad;                // low-rank K of the GEMM: 0, 32 (64-byte swizzle) or 64 (128-byte)
  int f16;                     // 1: the main loop is fp16 x fp16 (Lloyd-Max operand, decoded
                               //    residual), tmap_a / tmap_b are fp16 [M|N, K], no scales
  int64_t katoms;
  uint32_t* err;
};

cudaError_t launch_quantize_rows(const QuantParams& p, bool debug_xt, int num_sms,
                                 cudaStream_t st);
cudaError_t launch_encode_f32(const float* V, int M, int K, uint8_t* codes, uint8_t* scales,
                              cudaStream_t st, double lp = 0.0);
cudaError_t launch_lowrank_u(const LowRankParams& p, cudaStream_t st, bool dependent = true);
// kind: 0 none, 1 Kronecker; dependent: launched as a programmatic dependent of the previous
// kernel in the stream (the statistics kernel)
cudaError_t launch_quantize_chunks(const ChunkParams& p, int kind, bool center, bool debug_xt,
                                   bool dependent, int num_sms, cudaStream_t st);
// debug: one warp waits limit_ns on a barrier nothing completes, then sets the timeout bit
cudaError_t launch_wait_never(uint32_t* err, uint64_t limit_ns, cudaStream_t st);
// LayerNorm front-end, offline: l1gt = diag(gamma) (l1t hi + lo) as hi / lo rows,
// cg = gamma^T L1', cb = beta^T L1' (float64 sums in fixed order).
cudaError_t launch_ln_fold(const uint16_t* l1t, const float* gamma, const float* beta, int K,
                           uint16_t* l1gt, float* cg, float* cb, cudaStream_t st);
cudaError_t launch_gemm(const GemmParams& p, bool out_bf16, int num_sms, cudaStream_t st);
int gemm_tile_n();

}  // namespace kq
