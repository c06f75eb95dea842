// Memory layouts of the prepared-weights buffer and of the activation workspace.
//
// Block scales (one E8M0 byte per 32 elements along K) are stored in the layout the
// block-scaled tensor-core MMA consumes: rows are grouped by 128 and the K blocks by 4;
// each (128-row group, 4-block group) is one 512-byte atom in which the byte of
// (row r, block b) sits at  (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4).
// Atoms of one row group are consecutive along K, so the scales of one 128-row x
// 256-element GEMM tile are one contiguous 1 KB run. The K-block count is padded to a
// multiple of 8 (whole 256-element GEMM k-tiles); padding scales are written as 0.
#pragma once
#include <cstddef>
#include <cstdint>

namespace kq {

constexpr int kBlock = 32;          // MXFP4 block size along K
constexpr int kTileK = 256;         // FP4 elements per GEMM k-tile (128 bytes per row)
constexpr int kRankPad = 64;        // low-rank dimension as stored (rank <= 64)
constexpr int kUCols = 2 * kRankPad;         // U-kernel MMA width: L1' hi, L1' lo
constexpr int kUSplitMax = 8;                // largest split of K in the U kernel
constexpr int kHdrBytes = 256;               // workspace header: the device error word
constexpr size_t kAlign = 1024;

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// number of 4-block atoms per 128-row group for a given K
__host__ __device__ constexpr int64_t sf_katoms(int64_t K) { return 2 * cdiv(K, kTileK); }
__host__ __device__ constexpr size_t sf_bytes(int64_t rows_pad, int64_t K) {
  return static_cast<size_t>(rows_pad / 128) * static_cast<size_t>(sf_katoms(K)) * 512u;
}
__host__ __device__ __forceinline__ size_t sf_offset(int64_t row, int64_t kb, int64_t katoms) {
  return static_cast<size_t>(row / 128) * static_cast<size_t>(katoms) * 512u +
         static_cast<size_t>(kb / 4) * 512u + static_cast<size_t>(row % 32) * 16u +
         static_cast<size_t>((row % 128) / 32) * 4u + static_cast<size_t>(kb % 4);
}

// Physical byte offset of logical byte `off` in a buffer written by a TMA load with the
// 64-byte swizzle (16-byte chunk index XOR address bits 7..8); buffer 512-byte aligned.
__host__ __device__ __forceinline__ uint32_t swz64(uint32_t off) {
  return off ^ (((off >> 7) & 3u) << 4);
}

// RPBH table staged by the quantize kernel: uint16 source offsets (64-byte swizzled row
// byte offsets of perm[k], stored at the swizzled position of element k), then per
// 32-element block four 32-bit words whose nibble j of word w has bit 3 set when
// sign[32 b + 8 w + j] < 0 (the code's sign bit).
__host__ __device__ constexpr size_t qtab_bytes(int64_t K) {
  return static_cast<size_t>(K) * 2 + static_cast<size_t>(K / 32) * 16;
}

// LayerNorm table of the quantize kernel (shared-memory image, one bulk copy):
//  * K/32 lines of 256 bytes, line b = gamma (bytes 0..127) and beta (128..255) of the 32
//    values that block b of the transform input holds (for RPBH the gathered channels
//    perm[32 b + j]), each half as 8 chunks of 16 bytes, chunk c stored at c ^ (b % 8);
//  * RPBH only: K/32 lines of 128 bytes, gamma of channels 32 b .. 32 b + 31 in the same
//    chunk order (the statistics pass reads the row unpermuted);
//  * 16 bytes: mean_k beta_k as a float64, then 8 zero bytes.
__host__ __device__ constexpr size_t ln_table_bytes(int64_t K, int kind) {
  return static_cast<size_t>(K) * 8 + (kind == 2 ? static_cast<size_t>(K) * 4 : 0) + 16;
}
__host__ __device__ constexpr uint32_t ln_chunk_off(uint32_t b, uint32_t c) {
  return 16u * (c ^ (b & 7u));
}

struct WeightsLayout {
  int64_t K = 0, N = 0, rank = 0, rp = 0, n_pad = 0;
  bool center = false;
  int kind = 0;
  size_t rcodes = 0;   // uint8 [N, K/2]     residual codes (R^T, K-major)
  size_t rsf = 0;      // uint8 tiled        residual scales, rows padded (see n_pad)
  size_t l2t = 0;      // fp16  [N, rp]      L2^T (K-major B operand of the low-rank MMA)
  size_t l1t = 0;      // bf16  [kUCols, K]  rows 0..63 L1'^T hi, 64..127 lo
  size_t c1 = 0;       // f32   [rp]         1^T (L1' hi + lo)
  size_t s = 0;        // f32   [N]          1^T W
  size_t perm = 0;     // int32 [K]          RPBH gather indices
  size_t sgn = 0;      // f32   [K]          RPBH sign[k] / sqrt(32)
  size_t qtab = 0;     // uint8 [K*2 + K/32*16] RPBH table as the quantize kernel stages it
  size_t lng = 0;      // f32   [K]          LayerNorm gamma (front-end on)
  size_t lnb = 0;      // f32   [K]          LayerNorm beta
  size_t lntab = 0;    // the quantize kernel's LayerNorm table, as it is staged in shared
                       //   memory (ln_table_bytes)
  size_t l1gt = 0;     // bf16  [kUCols, K]  diag(gamma) L1' as hi / lo rows (front-end, rank > 0)
  size_t cg = 0;       // f32   [rp]         gamma^T L1'
  size_t cb = 0;       // f32   [rp]         beta^T L1'
  size_t rf16 = 0;     // fp16  [N, K]       residual decoded to fp16 (Lloyd-Max activations)
  size_t total = 0;

  __host__ __device__ static WeightsLayout make(int64_t K, int64_t N, int64_t rank, bool center,
                                                int kind, bool ln = false, bool lut = false) {
    WeightsLayout L;
    L.K = K; L.N = N; L.rank = rank; L.rp = rank > 0 ? kRankPad : 0; L.center = center;
    L.kind = kind;
    // 192-wide GEMM tiles read two 128-row scale atoms starting at floor(n0 / 128): keep one
    // spare (zero) atom after the last real one
    L.n_pad = cdiv(N, 128) * 128 + 128;
    size_t o = 256;  // header
    L.rcodes = o; o = align_up(o + static_cast<size_t>(N) * (K / 2), kAlign);
    L.rsf = o;    o = align_up(o + sf_bytes(L.n_pad, K), kAlign);
    L.l2t = o;    o = align_up(o + static_cast<size_t>(N) * L.rp * 2, kAlign);
    L.l1t = o;    o = align_up(o + (L.rp ? static_cast<size_t>(kUCols) * K * 2 : 0), kAlign);
    L.c1 = o;     o = align_up(o + static_cast<size_t>(L.rp) * 4, kAlign);
    L.s = o;      o = align_up(o + static_cast<size_t>(N) * 4, kAlign);
    L.perm = o;   o = align_up(o + (kind == 2 ? static_cast<size_t>(K) * 4 : 0), kAlign);
    L.sgn = o;    o = align_up(o + (kind == 2 ? static_cast<size_t>(K) * 4 : 0), kAlign);
    L.qtab = o;   o = align_up(o + (kind == 2 ? qtab_bytes(K) : 0), kAlign);
    L.lng = o;    o = align_up(o + (ln ? static_cast<size_t>(K) * 4 : 0), kAlign);
    L.lnb = o;    o = align_up(o + (ln ? static_cast<size_t>(K) * 4 : 0), kAlign);
    L.lntab = o;  o = align_up(o + (ln ? ln_table_bytes(K, kind) : 0), kAlign);
    const bool lr = ln && L.rp;
    L.l1gt = o;   o = align_up(o + (lr ? static_cast<size_t>(kUCols) * K * 2 : 0), kAlign);
    L.cg = o;     o = align_up(o + (lr ? static_cast<size_t>(L.rp) * 4 : 0), kAlign);
    L.cb = o;     o = align_up(o + (lr ? static_cast<size_t>(L.rp) * 4 : 0), kAlign);
    L.rf16 = o;   o = align_up(o + (lut ? static_cast<size_t>(N) * K * 2 : 0), kAlign);
    L.total = o;
    return L;
  }
};

// Split of the K reduction in the U kernel (a power of two <= 8): enough CTAs for a full
// GPU when M is small. The splits of one 128-row tile form a thread-block cluster.
__host__ __device__ constexpr int u_split(int64_t M, int64_t K) {
  const int64_t mt = cdiv(M, 128), kt = cdiv(K, 64);
  int s = 1;
  while (s < kUSplitMax && mt * (2 * s) <= 148 && 2 * (2 * s) <= kt) s *= 2;
  return s;
}

struct ActLayout {
  int64_t M = 0, m_pad = 0, K = 0, rp = 0;
  bool lut = false;    // Lloyd-Max activations: codes holds the fp16 operand, no sf
  size_t err = 0;      // uint32 device error word
  size_t codes = 0;    // uint8 [M, K/2] (MXFP4) or fp16 [M, K] (Lloyd-Max operand)
  size_t sf = 0;       // uint8 tiled, rows padded to 128 (MXFP4 only)
  size_t mu = 0;       // f32 [m_pad]
  size_t mulo = 0;     // f32 [m_pad] fp32(mu - fp32(mu)) (Kronecker / no-transform path)
  size_t u = 0;        // fp16 [M, rp]
  size_t lnm = 0;      // f32 [m_pad] LayerNorm mean of x (front-end on)
  size_t lnr = 0;      // f32 [m_pad] LayerNorm 1/sqrt(v + eps)
  size_t sig = 0;      // f32 [m_pad] per-token sigma (Lloyd-Max activations)
  size_t total = 0;

  __host__ __device__ static ActLayout make(int64_t M, int64_t K, int64_t rank, bool ln = false,
                                            bool lut = false) {
    ActLayout L;
    L.M = M; L.K = K; L.rp = rank > 0 ? kRankPad : 0; L.lut = lut;
    L.m_pad = cdiv(M, 128) * 128;
    size_t o = 0;
    L.err = o;    o = kHdrBytes;
    L.codes = o;  o = align_up(o + static_cast<size_t>(M) * (lut ? K * 2 : K / 2), kAlign);
    L.sf = o;     o = align_up(o + (lut ? 0 : sf_bytes(L.m_pad, K)), kAlign);
    L.mu = o;     o = align_up(o + static_cast<size_t>(L.m_pad) * 4, kAlign);
    L.mulo = o;   o = align_up(o + static_cast<size_t>(L.m_pad) * 4, kAlign);
    L.u = o;      o = align_up(o + static_cast<size_t>(M) * L.rp * 2, kAlign);
    L.lnm = o;    o = align_up(o + (ln ? static_cast<size_t>(L.m_pad) * 4 : 0), kAlign);
    L.lnr = o;    o = align_up(o + (ln ? static_cast<size_t>(L.m_pad) * 4 : 0), kAlign);
    L.sig = o;    o = align_up(o + (lut ? static_cast<size_t>(L.m_pad) * 4 : 0), kAlign);
    L.total = o;
    return L;
  }
};

}  // namespace kq
