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
//    RPBH(X) = X P H D), or a per-channel multiply by SmoothQuant inverse scales (the
//    comparator of KroQuant section 02). MXFP4 encoding as in encode.cuh (KroQuant
//    section 03), or (template LUT) the nearest level of a 16-level Lloyd-Max codebook
//    of N(0, 1) for Xt / sigma with sigma the RMS of the centred token (OrbitQuant
//    section 03; CentriQ abstract: the per-token scale in closed form), stored as the
//    fp16 operand the contraction takes.
//  * k_lowrank_u -- U = X L1' - mu c1 (SVDQuant explainer, section 3: the low-rank branch
//    runs on the high-precision input) as a tcgen05 bf16 GEMM: TMA loads 128x64 tiles of
//    X and of [L1'_hi; L1'_lo], the MMA accumulates 128 x 128 in TMEM, the epilogue forms
//    hi + lo - mu c1 (mu from the quantize kernel) and stores fp16 (16-bit branch). For
//    small M the K reduction is split over a cluster and reduced in distributed smem.
//  * LayerNorm front-end (y = (x - m) rstd gamma + beta per token, ahead of the layer):
//    the quantize kernel forms m, rstd and mean(y) from the staged row (a second, centred
//    pass gives the variance) and normalises each block before centring it; the low-rank
//    kernel still streams raw x, against diag(gamma) L1', and its epilogue applies
//    y L1' = rstd (x diag(gamma) L1') - rstd m gamma^T L1' + beta^T L1'.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kq_internal.cuh"
#include "packed.cuh"

namespace kq {

// ----------------------------------------------------------------------------------
// helpers
// ----------------------------------------------------------------------------------
__device__ __forceinline__ double warp_sum_f64(double x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ----------------------------------------------------------------------------------
// k_quantize_rows
// ----------------------------------------------------------------------------------
// Groups of R consecutive token rows; each row is staged by TMA (64-byte swizzle, one
// 64-byte line per 32-element block) into its own 512-byte aligned slot of a ring of up
// to 4 group buffers; one consumer lane per block. The CTA walks groups blockIdx.x,
// +gridDim.x, ... Arithmetic runs on fp32 pairs (Blackwell f32x2 FMA/ADD/SUB/MUL), each
// lane rounded like the scalar instruction.

// Kronecker apply on pairs: v2[4i + jp] = (x[8i+2jp], x[8i+2jp+1]);
// T[i][l] = sum_j x[8i+j] B[j][l] with Bp[4j + lp] = (B[j][2lp], B[j][2lp+1]);
// Y[k][l] = sum_i A[i][k] T[i][l] with Ap[4i + k] = (A[i][k], A[i][k]).
__device__ __forceinline__ void kron_apply2(uint64_t (&v2)[16], const uint64_t (&Ap)[16],
                                            const uint64_t (&Bp)[32]) {
  uint64_t t2[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t acc[4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = (j & 1) ? f2hi(v2[4 * i + j / 2]) : f2lo(v2[4 * i + j / 2]);
      const uint64_t xx = f2pack(x, x);
#pragma unroll
      for (int lp = 0; lp < 4; ++lp)
        acc[lp] = j == 0 ? fmul2(xx, Bp[lp]) : ffma2(xx, Bp[4 * j + lp], acc[lp]);
    }
#pragma unroll
    for (int lp = 0; lp < 4; ++lp) t2[4 * i + lp] = acc[lp];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int lp = 0; lp < 4; ++lp) {
      uint64_t acc = fmul2(Ap[k], t2[lp]);
#pragma unroll
      for (int i = 1; i < 4; ++i) acc = ffma2(Ap[4 * i + k], t2[4 * i + lp], acc);
      v2[4 * k + lp] = acc;
    }
}

// kron_apply2 whose second stage starts from bias2[4k + lp] instead of 0: adds a constant
// per output element in the same pass (used to apply a per-token correction -m (1^T P)).
__device__ __forceinline__ void kron_apply2_bias(uint64_t (&v2)[16], const uint64_t (&Ap)[16],
                                                 const uint64_t (&Bp)[32], const uint64_t (&bias2)[16]) {
  uint64_t t2[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t acc[4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = (j & 1) ? f2hi(v2[4 * i + j / 2]) : f2lo(v2[4 * i + j / 2]);
      const uint64_t xx = f2pack(x, x);
#pragma unroll
      for (int lp = 0; lp < 4; ++lp)
        acc[lp] = j == 0 ? fmul2(xx, Bp[lp]) : ffma2(xx, Bp[4 * j + lp], acc[lp]);
    }
#pragma unroll
    for (int lp = 0; lp < 4; ++lp) t2[4 * i + lp] = acc[lp];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int lp = 0; lp < 4; ++lp) {
      uint64_t acc = ffma2(Ap[k], t2[lp], bias2[4 * k + lp]);
#pragma unroll
      for (int i = 1; i < 4; ++i) acc = ffma2(Ap[4 * i + k], t2[4 * i + lp], acc);
      v2[4 * k + lp] = acc;
    }
}

// Unnormalised 32-point Walsh-Hadamard transform (Sylvester order) on pairs.
__device__ __forceinline__ void fwht32_2(uint64_t (&v2)[16]) {
#pragma unroll
  for (int hp = 1; hp < 16; hp <<= 1)          // element strides 2, 4, 8, 16
#pragma unroll
    for (int p = 0; p < 16; ++p)
      if ((p & hp) == 0) {
        const uint64_t a = v2[p], b = v2[p + hp];
        v2[p] = fadd2(a, b);
        v2[p + hp] = fsub2(a, b);
      }
#pragma unroll
  for (int p = 0; p < 16; ++p) {                // element stride 1: inside each pair
    float a, b;
    f2unpack(v2[p], a, b);
    v2[p] = f2pack(a + b, a - b);
  }
}

__device__ __forceinline__ float amax32_2(const uint64_t (&v2)[16]) {
  float m = 0.f;
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    float a, b;
    f2unpack(v2[p], a, b);
    m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
  }
  return m;
}

// codes of v2 * f (f a scale whose product with each value is the value / 2^e)
__device__ __forceinline__ void encode_scaled2(const uint64_t (&v2)[16], float f, uint32_t (&c)[4]) {
  const uint64_t ff = f2pack(f, f);
#pragma unroll
  for (int w = 0; w < 4; ++w)
    c[w] = cvt_e2m1x8(fmul2(v2[4 * w], ff), fmul2(v2[4 * w + 1], ff), fmul2(v2[4 * w + 2], ff),
                      fmul2(v2[4 * w + 3], ff));
}


// Transform + encode of one 32-element block (row r of the ring slot, block b). Writes the
// codes (or, in debug mode, the transformed values) and returns the scale byte.
// CENTER: 0 off, 1 centring, 2 LayerNorm then centring of the normalised token.
// LUT: Lloyd-Max codebook out (ln = sigma, 1/sigma) instead of MXFP4.
template <int KIND, int CENTER, bool DEBUG_XT, bool LUT>
__device__ __forceinline__ uint32_t quantize_block(const QuantParams& p, const uint64_t (&Ap)[16],
                                                   const uint64_t (&Bp)[32], const uint8_t* rowb,
                                                   const uint8_t* tables, const uint8_t* lntab,
                                                   int row, int b, float mu_hi, float mu_lo,
                                                   float4 ln) {
  const float rs = 0.17677669529663687f;   // fp32(1 / sqrt(32))
  uint64_t v2[16];
  if (KIND == 2) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 ix = *reinterpret_cast<const uint4*>(
          tables + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
      const uint32_t w4[4] = {ix.x, ix.y, ix.z, ix.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint16_t h0 = *reinterpret_cast<const uint16_t*>(rowb + (w4[t] & 0xFFFFu));
        const uint16_t h1 = *reinterpret_cast<const uint16_t*>(rowb + (w4[t] >> 16));
        v2[4 * c + t] = f2pack(__uint_as_float(static_cast<uint32_t>(h0) << 16),
                               __uint_as_float(static_cast<uint32_t>(h1) << 16));
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 q = *reinterpret_cast<const uint4*>(rowb + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
      v2[4 * c + 0] = bf16x2_to_f2(q.x);
      v2[4 * c + 1] = bf16x2_to_f2(q.y);
      v2[4 * c + 2] = bf16x2_to_f2(q.z);
      v2[4 * c + 3] = bf16x2_to_f2(q.w);
    }
  }
  if (KIND == 3) {
    // per-channel inverse scales of this block: 128-byte line b of the table, 16-byte
    // chunk c stored at chunk c ^ (b % 8) (consecutive lanes read distinct banks)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 f = *reinterpret_cast<const float4*>(
          tables + static_cast<uint32_t>(b) * 128u + 16u * (static_cast<uint32_t>(c) ^ (static_cast<uint32_t>(b) & 7u)));
      v2[2 * c] = fmul2(v2[2 * c], f2pack(f.x, f.y));
      v2[2 * c + 1] = fmul2(v2[2 * c + 1], f2pack(f.z, f.w));
    }
  }
  if (CENTER) {
    const uint64_t mh = f2pack(mu_hi, mu_hi), ml = f2pack(mu_lo, mu_lo);
#pragma unroll
    for (int q = 0; q < 16; ++q) v2[q] = fsub2(fsub2(v2[q], mh), ml);
  }
  if (CENTER == 2) {
    // y = (x - m) rstd gamma + beta, then y - mean(y) (ln = rstd, mean hi, mean lo)
    const uint64_t rr = f2pack(ln.x, ln.x);
    const uint64_t yh = f2pack(ln.y, ln.y), yl = f2pack(ln.z, ln.z);
    const uint8_t* line = lntab + static_cast<uint32_t>(b) * 256u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t o = ln_chunk_off(static_cast<uint32_t>(b), static_cast<uint32_t>(c));
      const float4 g = *reinterpret_cast<const float4*>(line + o);
      const float4 be = *reinterpret_cast<const float4*>(line + 128u + o);
      v2[2 * c] = fsub2(fsub2(ffma2(fmul2(v2[2 * c], rr), f2pack(g.x, g.y), f2pack(be.x, be.y)), yh), yl);
      v2[2 * c + 1] =
          fsub2(fsub2(ffma2(fmul2(v2[2 * c + 1], rr), f2pack(g.z, g.w), f2pack(be.z, be.w)), yh), yl);
    }
  }
  if (KIND == 1) kron_apply2(v2, Ap, Bp);
  if (KIND == 2) fwht32_2(v2);
  const uint32_t* signs = reinterpret_cast<const uint32_t*>(tables + static_cast<size_t>(p.K) * 2);
  if (DEBUG_XT) {
    if (KIND == 2) {
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float a, c2;
        f2unpack(v2[q], a, c2);
        const uint32_t mw = signs[4 * b + q / 4];
        const uint32_t s0 = (mw >> (4 * (2 * (q % 4)) + 3)) & 1u;
        const uint32_t s1 = (mw >> (4 * (2 * (q % 4) + 1) + 3)) & 1u;
        v2[q] = f2pack(__uint_as_float(__float_as_uint(a * rs) ^ (s0 << 31)),
                       __uint_as_float(__float_as_uint(c2 * rs) ^ (s1 << 31)));
      }
    }
    float4* o = reinterpret_cast<float4*>(p.xt + static_cast<size_t>(row) * p.K + b * kBlock);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      o[q] = make_float4(f2lo(v2[2 * q]), f2hi(v2[2 * q]), f2lo(v2[2 * q + 1]), f2hi(v2[2 * q + 1]));
    return 0u;
  }
  if (LUT) {
    // |Xt| / sigma against the thresholds (a magnitude on a threshold takes the larger
    // level), the level times sigma rounded to fp16, the sign of Xt (RPBH: of y times the
    // channel sign) set on the result
    const float cinv = KIND == 2 ? rs * ln.y : ln.y;
    float mg[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mg[i] = ln.x * p.lut_mag[i];
    uint32_t out[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      float a, c2;
      f2unpack(v2[q], a, c2);
      uint32_t s0 = __float_as_uint(a) >> 31, s1 = __float_as_uint(c2) >> 31;
      if (KIND == 2) {
        const uint32_t mw = signs[4 * b + q / 4];
        s0 ^= (mw >> (4 * (2 * (q % 4)) + 3)) & 1u;
        s1 ^= (mw >> (4 * (2 * (q % 4) + 1) + 3)) & 1u;
      }
      const float ta = fabsf(a) * cinv, tb = fabsf(c2) * cinv;
      float va = mg[0], vb = mg[0];
#pragma unroll
      for (int j = 0; j < 7; ++j) {
        va = ta >= p.lut_thr[j] ? mg[j + 1] : va;
        vb = tb >= p.lut_thr[j] ? mg[j + 1] : vb;
      }
      const __half2 h = __floats2half2_rn(va, vb);
      out[q] = *reinterpret_cast<const uint32_t*>(&h) | (s0 << 15) | (s1 << 31);
    }
    uint4* o = reinterpret_cast<uint4*>(p.a16 + static_cast<size_t>(row) * p.K + b * kBlock);
#pragma unroll
    for (int v = 0; v < 4; ++v) o[v] = make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2], out[4 * v + 3]);
    return 0u;
  }
  uint32_t c[4];
  uint32_t sbyte;
  if (KIND == 2) {
    // Xt = y * rs * sign. amax(y * rs) = fl(amax(y) * rs) (rounding is monotonic), and
    // fl(y * rs) / 2^e = fl(y * (rs / 2^e)) (power-of-two scaling commutes with rounding
    // for normal results); the sign flips the code's sign bit.
    sbyte = mx_scale_byte(amax32_2(v2) * rs);
    if (sbyte > 0) {
      encode_scaled2(v2, rs * mx_inv_scale(sbyte), c);
    } else {
      const uint64_t rr = f2pack(rs, rs);       // tiny block: keep the two-step rounding
#pragma unroll
      for (int q = 0; q < 16; ++q) v2[q] = fmul2(v2[q], rr);
      encode_scaled2(v2, mx_inv_scale(sbyte), c);
    }
    const uint4 sg = *reinterpret_cast<const uint4*>(signs + 4 * b);
    c[0] ^= sg.x; c[1] ^= sg.y; c[2] ^= sg.z; c[3] ^= sg.w;
  } else {
    sbyte = mx_scale_byte(amax32_2(v2));
    encode_scaled2(v2, mx_inv_scale(sbyte), c);
  }
  *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * (p.K / 2) + b * 16) =
      make_uint4(c[0], c[1], c[2], c[3]);
  return sbyte;
}

// Scale bytes of 4 consecutive blocks held by 4 consecutive lanes (lane % 4 == 0 is the
// first) become one 32-bit word; or, when K/32 is not a multiple of 4, single bytes.
__device__ __forceinline__ void store_scales(const QuantParams& p, bool valid, int row, int b,
                                             int nb, int nb_pad, uint32_t sbyte) {
  const int lane = threadIdx.x & 31;
  if ((nb & 3) == 0) {
    const uint32_t w = sbyte | (__shfl_down_sync(0xffffffffu, sbyte, 1) << 8) |
                       (__shfl_down_sync(0xffffffffu, sbyte, 2) << 16) |
                       (__shfl_down_sync(0xffffffffu, sbyte, 3) << 24);
    if (valid && (lane & 3) == 0) {
      *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, b, p.katoms)) = w;
      if (b + 4 == nb)                                   // zero the padding blocks of the row
        for (int bb = nb; bb < nb_pad; bb += 4)
          *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, bb, p.katoms)) = 0u;
    }
  } else if (valid) {
    p.sf[sf_offset(row, b, p.katoms)] = static_cast<uint8_t>(sbyte);
    if (b == nb - 1)
      for (int bb = nb; bb < nb_pad; ++bb) p.sf[sf_offset(row, bb, p.katoms)] = 0;
  }
}

// Persistent; every warp is its own pipeline. The work is cut into units of u consecutive
// token rows (u chosen so that u * K/32 blocks fill the lanes of a warp evenly); unit j
// belongs to CTA j % gridDim.x, and a CTA's units go round-robin to its warps. Each warp
// owns a ring of S slots in shared memory and issues its own TMA loads into them (one
// 512-byte aligned, 64-byte swizzled slot row per token): when it has finished a unit it
// refills that slot with its unit S further on, so the next units are in flight while it
// computes and no warp ever waits for another. RPBH gather offsets and sign masks arrive
// once per CTA, as one bulk copy of a table prepared with the weights; the Kronecker
// factors live in registers. Centring: the warp forms each row's mean (fp32 block sums,
// fp64 across blocks), then all u * K/32 blocks of the unit are spread over the lanes.
template <int KIND, int CENTER, bool DEBUG_XT, bool LUT>
__global__ void __launch_bounds__(KIND == 1 ? 32 * kQMaxWarpsKron : 32 * kQMaxWarps, 1)
k_quantize_rows(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NW = p.consumer_warps;
  const int nb = p.K / kBlock;
  const int nb_pad = static_cast<int>(p.katoms) * 4;
  const int u = p.unit_rows;
  const int S = p.nbufs;
  const uint32_t rstride = p.row_stride;
  const uint32_t slot_bytes = static_cast<uint32_t>(u) * rstride;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);             // [NW * S]
  uint64_t* tabbar = full + kQMaxWarps * kQMaxStages;
  float2* wmu = reinterpret_cast<float2*>(smem + kQMuOff) + 32 * warp;   // this warp's means
  float4* wln = reinterpret_cast<float4*>(smem + kQLnOff) + 32 * warp;   // LayerNorm row terms
  const uint8_t* lntab = smem + p.lntab_off;
  uint8_t* tables = smem + p.tables_off;
  uint8_t* wbufs = smem + p.bufs_off + static_cast<size_t>(warp) * S * slot_bytes;
  const int64_t units = cdiv(p.M, u);
  const int G = static_cast<int>(gridDim.x);
  const int64_t nl = (units - blockIdx.x + G - 1) / G;             // this CTA's units
  uint64_t* wfull = full + warp * S;
  // The device error word starts at zero for this call. This grid is launched in plain
  // stream order (after every kernel of the previous call has finished), and a kernel of
  // this call can set the word only when one of its waits has run 2 s, long after CTA 0
  // has started, so clearing it here cannot lose an error.
  if (blockIdx.x == 0 && tid == 0 && p.err != nullptr && !p.keep_err) *p.err = 0u;

  uint64_t Ap[16], Bp[32];
  if (KIND == 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) Ap[i] = p.Ap[i];
#pragma unroll
    for (int i = 0; i < 32; ++i) Bp[i] = p.Bp[i];
  }

  // load unit l (a multiple of NW away from this warp's first) into slot s
  auto issue = [&](int64_t l, int s) {
    const int64_t row0 = (l * G + blockIdx.x) * u;
    const int rows = static_cast<int>(min(static_cast<int64_t>(u), p.M - row0));
    uint8_t* dst = wbufs + static_cast<size_t>(s) * slot_bytes;
    mbar_arrive_expect_tx(&wfull[s], static_cast<uint32_t>(rows) * nb * 64u);
    for (int r = 0; r < rows; ++r)
      for (int c = 0; c < nb; c += p.box_lines)
        tma_load_2d(dst + static_cast<size_t>(r) * rstride + static_cast<size_t>(c) * 64u,
                    &p.tmap_x, 0, static_cast<int32_t>((row0 + r) * nb + c), &wfull[s]);
  };

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&wfull[s], 1);
    if (warp == 0) mbar_init(tabbar, 1);
    fence_mbar_init();
    if (warp == 0) {
      prefetch_tmap(&p.tmap_x);
      if (KIND == 2 || CENTER == 2) {
        mbar_arrive_expect_tx(tabbar, (KIND == 2 ? p.qtab_bytes : 0u) +
                                          (CENTER == 2 ? p.lntab_bytes : 0u));
        if (KIND == 2) bulk_load(tables, p.qtab, p.qtab_bytes, tabbar);
        if (CENTER == 2) bulk_load(smem + p.lntab_off, p.lntab, p.lntab_bytes, tabbar);
      }
    }
    for (int s = 0; s < S; ++s)
      if (warp + static_cast<int64_t>(s) * NW < nl) issue(warp + static_cast<int64_t>(s) * NW, s);
  }
  if (KIND == 3) {
    // per-channel inverse scales into 128-byte lines (one per block), chunk-swizzled
    for (int k4 = tid; k4 < p.K / 4; k4 += blockDim.x) {
      const uint32_t b = static_cast<uint32_t>(k4 / 8), c = static_cast<uint32_t>(k4 % 8);
      *reinterpret_cast<float4*>(tables + b * 128u + 16u * (c ^ (b & 7u))) =
          reinterpret_cast<const float4*>(p.inv_s)[k4];
    }
  }
  __syncthreads();                                                  // tabbar initialised
  grid_dep_launch();                       // the low-rank / GEMM kernel may start its prologue

  bool ok = true;
  if (KIND == 2 || CENTER == 2)
    ok = __all_sync(0xffffffffu, mbar_wait(tabbar, 0, p.err, KQ_DEV_ERR_TIMEOUT_FULL));
  int64_t k = 0;
  for (int64_t l = warp; ok && l < nl; l += NW, ++k) {
    const int s = static_cast<int>(k % S);
    ok = __all_sync(0xffffffffu,
                    mbar_wait(&wfull[s], static_cast<uint32_t>(k / S) & 1u, p.err, KQ_DEV_ERR_TIMEOUT_FULL));
    if (!ok) break;
    const uint8_t* ub = wbufs + static_cast<size_t>(s) * slot_bytes;
    const int64_t row0 = (l * G + blockIdx.x) * u;
    const int rows = static_cast<int>(min(static_cast<int64_t>(u), p.M - row0));
    if (CENTER || LUT) {
      for (int r = 0; r < rows; ++r) {
        const uint8_t* rowb = ub + static_cast<size_t>(r) * rstride;
        double part = 0.0;
        for (int b = lane; CENTER && b < nb; b += 32) {
          uint64_t acc = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(rowb + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
            const uint64_t s0 = fadd2(bf16x2_to_f2(q.x), bf16x2_to_f2(q.y));
            const uint64_t s1 = fadd2(bf16x2_to_f2(q.z), bf16x2_to_f2(q.w));
            acc = c == 0 ? fadd2(s0, s1) : fadd2(acc, fadd2(s0, s1));
          }
          part += static_cast<double>(f2lo(acc) + f2hi(acc));
        }
        const double mu64 = CENTER ? warp_sum_f64(part) / static_cast<double>(p.K) : 0.0;
        const float mu_hi = static_cast<float>(mu64);
        const float mu_lo = static_cast<float>(mu64 - static_cast<double>(mu_hi));
        if (CENTER == 2) {
          // second pass over the staged row, centred: sum d^2 and sum d gamma with
          // d = (x - m_hi) - m_lo (fp32 per block, fp64 across blocks)
          const uint64_t mh = f2pack(mu_hi, mu_hi), ml = f2pack(mu_lo, mu_lo);
          const uint8_t* gbase = KIND == 2 ? lntab + static_cast<size_t>(p.K) * 8 : lntab;
          const uint32_t gstride = KIND == 2 ? 128u : 256u;
          double pv = 0.0, pg = 0.0;
          for (int b = lane; b < nb; b += 32) {
            uint64_t av = 0, ag = 0;
            const uint8_t* gl = gbase + static_cast<uint32_t>(b) * gstride;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 q = *reinterpret_cast<const uint4*>(rowb + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
              const float4 g0 = *reinterpret_cast<const float4*>(
                  gl + ln_chunk_off(static_cast<uint32_t>(b), static_cast<uint32_t>(2 * c)));
              const float4 g1 = *reinterpret_cast<const float4*>(
                  gl + ln_chunk_off(static_cast<uint32_t>(b), static_cast<uint32_t>(2 * c + 1)));
              const uint64_t d0 = fsub2(fsub2(bf16x2_to_f2(q.x), mh), ml);
              const uint64_t d1 = fsub2(fsub2(bf16x2_to_f2(q.y), mh), ml);
              const uint64_t d2 = fsub2(fsub2(bf16x2_to_f2(q.z), mh), ml);
              const uint64_t d3 = fsub2(fsub2(bf16x2_to_f2(q.w), mh), ml);
              av = ffma2(d0, d0, av); av = ffma2(d1, d1, av); av = ffma2(d2, d2, av); av = ffma2(d3, d3, av);
              ag = ffma2(d0, f2pack(g0.x, g0.y), ag); ag = ffma2(d1, f2pack(g0.z, g0.w), ag);
              ag = ffma2(d2, f2pack(g1.x, g1.y), ag); ag = ffma2(d3, f2pack(g1.z, g1.w), ag);
            }
            pv += static_cast<double>(f2lo(av)) + static_cast<double>(f2hi(av));
            pg += static_cast<double>(f2lo(ag)) + static_cast<double>(f2hi(ag));
          }
          const double var = warp_sum_f64(pv) / static_cast<double>(p.K);
          const double sdg = warp_sum_f64(pg);
          const double rstd = 1.0 / sqrt(var + p.ln_eps);
          const double mean_b = *reinterpret_cast<const double*>(lntab + p.lntab_bytes - 16u);
          const double my = rstd * sdg / static_cast<double>(p.K) + mean_b;
          const float my_hi = static_cast<float>(my);
          const float my_lo = static_cast<float>(my - static_cast<double>(my_hi));
          if (lane == 0) {
            wmu[r] = make_float2(mu_hi, mu_lo);
            wln[r] = make_float4(static_cast<float>(rstd), my_hi, my_lo, 0.f);
            p.mu[row0 + r] = my_hi;
            if (p.lnm != nullptr) {                  // null in the debug entry
              // a token with zero variance normalises to beta exactly: its low-rank input
              // is beta^T L1' - mean(y) c1, so the epilogue gets no rstd term for it
              p.lnm[row0 + r] = mu_hi;
              p.lnr[row0 + r] = var > 0.0 ? static_cast<float>(rstd) : 0.f;
            }
          }
        } else {
          if (LUT) {
            // sigma = RMS of the (centred) token, which the orthonormal rotation keeps:
            // sum d^2 with d = (x - m_hi) - m_lo, fp32 per block, fp64 across blocks
            const uint64_t mh = f2pack(mu_hi, mu_hi), ml = f2pack(mu_lo, mu_lo);
            double pv = 0.0;
            for (int b = lane; b < nb; b += 32) {
              uint64_t av = 0;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint4 q = *reinterpret_cast<const uint4*>(rowb + swz64(static_cast<uint32_t>(b) * 64u + 16u * c));
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const uint64_t d = CENTER ? fsub2(fsub2(bf16x2_to_f2(w4[t]), mh), ml) : bf16x2_to_f2(w4[t]);
                  av = ffma2(d, d, av);
                }
              }
              pv += static_cast<double>(f2lo(av)) + static_cast<double>(f2hi(av));
            }
            const double sg = sqrt(warp_sum_f64(pv) / static_cast<double>(p.K));
            const float sg32 = static_cast<float>(sg);
            const float inv32 = sg > 0.0 ? static_cast<float>(1.0 / sg) : 0.f;
            if (lane == 0) {
              wln[r] = make_float4(sg32, inv32, 0.f, 0.f);
              p.sig[row0 + r] = sg32;
            }
          }
          if (lane == 0) {
            wmu[r] = make_float2(mu_hi, mu_lo);
            p.mu[row0 + r] = mu_hi;
          }
        }
      }
      __syncwarp();
    } else if (lane < rows) {
      p.mu[row0 + lane] = 0.f;
    }
    // all blocks of the unit over the lanes: item i = (row i / nb, block i % nb)
    const int items = rows * nb;
    const int iters = (u * nb + 31) / 32;
    int r = 0, b = lane;
    while (b >= nb) { b -= nb; ++r; }
    for (int t = 0; t < iters; ++t) {
      const bool valid = 32 * t + lane < items;
      uint32_t sb = 0;
      if (valid) {
        float mh = 0.f, ml = 0.f;
        float4 lr = make_float4(0.f, 0.f, 0.f, 0.f);
        if (CENTER) { const float2 m = wmu[r]; mh = m.x; ml = m.y; }
        if (CENTER == 2 || LUT) lr = wln[r];
        sb = quantize_block<KIND, CENTER, DEBUG_XT, LUT>(p, Ap, Bp, ub + static_cast<size_t>(r) * rstride,
                                                    tables, lntab, static_cast<int>(row0 + r), b, mh,
                                                    ml, lr);
      }
      if (!DEBUG_XT && !LUT) store_scales(p, valid, static_cast<int>(row0 + r), b, nb, nb_pad, sb);
      b += 32;
      while (b >= nb) { b -= nb; ++r; }
    }
    // every lane is done with the slot: refill it with this warp's unit S further on
    __syncwarp();
    if (lane == 0 && l + static_cast<int64_t>(S) * NW < nl) {
      fence_async_smem();                   // generic reads of the slot before the async write
      issue(l + static_cast<int64_t>(S) * NW, s);
    }
  }
  // rows M .. m_pad-1 of the last 128-row group: zero scales (finite values for the GEMM)
  if (!DEBUG_XT) {
    const int wpr = nb_pad / 4;
    const int pad_rows = p.m_pad - p.M;
    const int nthr = NW * 32;
    for (int i = blockIdx.x * nthr + tid; i < pad_rows * wpr; i += G * nthr) {
      const int rr = p.M + i / wpr, w = i % wpr;
      if (!LUT) *reinterpret_cast<uint32_t*>(p.sf + sf_offset(rr, 4 * w, p.katoms)) = 0u;
      if (w == 0) {
        p.mu[rr] = 0.f;
        if (CENTER == 2) { p.lnm[rr] = 0.f; p.lnr[rr] = 0.f; }
        if (LUT) p.sig[rr] = 0.f;
      }
    }
  }
  // no TMA load may still be writing this CTA's shared memory when it exits: a warp
  // that stopped early (device error) drains its outstanding slots first
  if (!ok && lane == 0) {
    for (int64_t kk = k; kk < k + S; ++kk) {
      const int64_t ll = warp + kk * NW;
      if (ll >= nl) break;
      mbar_wait(&wfull[kk % S], static_cast<uint32_t>(kk / S) & 1u, nullptr, 0);
    }
  }
}

// ----------------------------------------------------------------------------------
// k_encode_f32 (debug): encoder alone on float32 rows, canonical outputs (plain OCP rule,
// or the robust l_p scale fit when lp > 0)
// ----------------------------------------------------------------------------------
__global__ void k_encode_f32(const float* __restrict__ V, int M, int K, uint8_t* __restrict__ codes,
                             uint8_t* __restrict__ scales, double lp) {
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
  const uint32_t sb = lp > 0.0 ? mx_encode32_lp(v, lp, c) : mx_encode32(v, c);
  *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = make_uint4(c[0], c[1], c[2], c[3]);
  scales[row * nb + b] = static_cast<uint8_t>(sb);
}

// ----------------------------------------------------------------------------------
// k_wait_never (debug): one warp waits, with the given limit, on an mbarrier that nothing
// arrives on. The wait runs out, sets KQ_DEV_ERR_TIMEOUT_FULL in the error word and the
// kernel returns: the path every kernel's bounded waits take when a stage never fills.
// ----------------------------------------------------------------------------------
__global__ void k_wait_never(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0, threadIdx.x == 0 ? err : nullptr, KQ_DEV_ERR_TIMEOUT_FULL, limit_ns);
  (void)__all_sync(0xffffffffu, ok);
}

cudaError_t launch_wait_never(uint32_t* err, uint64_t limit_ns, cudaStream_t st) {
  k_wait_never<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------------
// k_lowrank_u: U[m, 0..63] = X L1'_hi + X L1'_lo - mu[m] c1, stored as fp16
// ----------------------------------------------------------------------------------
// Grid (M/128, S), S in {1, 2, 4, 8}: CTA (mt, ks) accumulates the 128-row tile over its
// share of the K chunks. With S > 1 the S CTAs of a tile form a cluster: each stages its
// fp32 partial in its own shared memory, and CTA ks then sums rows [ks*128/S, ...) over
// all S partials (distributed shared memory, fixed order: deterministic).
namespace lowrank {
constexpr int kStages = 3;
constexpr int kTileM = 128;
constexpr int kChunkK = 64;                      // bf16 elements per stage (128 bytes)
constexpr uint32_t kABytes = kTileM * 128;       // 16 KB
constexpr uint32_t kBBytes = kUCols * 128;       // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + 1024;
// when the quantize kernel's shape leaves no room beside it, the ring is deeper
constexpr int kStagesDeep = 6;
constexpr uint32_t smem_bytes(int ns) { return 1024 + ns * kStageBytes + 1024; }
constexpr uint32_t kTmemCols = 128;
static_assert(kSmemBytes == kLowRankSmemBytes, "shared-memory footprint the quantize shape leaves room for");
}  // namespace lowrank

// fp16 pair of two U values, saturated at +-65504; `over` is set when either lies outside
// that range or is not a number (the caller reports it through the device error word)
__device__ __forceinline__ uint32_t f2_to_half2_sat(float a, float b, bool& over) {
  over |= !(fabsf(a) <= 65504.f) || !(fabsf(b) <= 65504.f);
  a = fminf(fmaxf(a, -65504.f), 65504.f);
  b = fminf(fmaxf(b, -65504.f), 65504.f);
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// one lane of the warp records a saturated U value in the error word
__device__ __forceinline__ void report_u_range(uint32_t* err, bool over) {
  if (__any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0 && err != nullptr)
    atomicOr(err, KQ_DEV_ERR_U_RANGE);
}

// One output of the U epilogue from the accumulated x L: acc - mu c1[j], or with the
// LayerNorm front-end (L = diag(gamma) L1') rstd acc - rstd m cg[j] + cb[j] - mu c1[j],
// which is y L1' - mean(y) c1 for y = LayerNorm(x). mu is the row's fp32 mean (0 when the
// layer does not centre).
struct URowTerms { float mu, rs, rm; };
__device__ __forceinline__ URowTerms u_row_terms(const LowRankParams& p, int row, float mu) {
  URowTerms t;
  t.mu = mu;
  t.rs = p.ln ? p.lnr[row] : 1.f;
  t.rm = p.ln ? t.rs * p.lnm[row] : 0.f;
  return t;
}
__device__ __forceinline__ float u_value(const LowRankParams& p, const URowTerms& t, float acc, int j) {
  if (p.ln) return fmaf(t.rs, acc, fmaf(-t.rm, p.cg[j], p.cb[j])) - t.mu * p.c1[j];
  return acc - t.mu * p.c1[j];
}

// Sum of the 64 bf16 values of one staged row piece (128 bytes, 128-byte swizzle, row rl of
// the tile): fp32 within each 32-element block (pairs, then the two halves), the two block
// sums added in float64.
__device__ __forceinline__ double chunk_row_sum(const uint8_t* tile, int rl) {
  const uint8_t* rowp = tile + static_cast<uint32_t>(rl) * 128u;
  double s = 0.0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint64_t acc = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 q = *reinterpret_cast<const uint4*>(
          rowp + 16u * ((static_cast<uint32_t>(4 * h + c)) ^ (static_cast<uint32_t>(rl) & 7u)));
      const uint64_t s0 = fadd2(bf16x2_to_f2(q.x), bf16x2_to_f2(q.y));
      const uint64_t s1 = fadd2(bf16x2_to_f2(q.z), bf16x2_to_f2(q.w));
      acc = c == 0 ? fadd2(s0, s1) : fadd2(acc, fadd2(s0, s1));
    }
    s += static_cast<double>(f2lo(acc) + f2hi(acc));
  }
  return s;
}

// The row mean as written for the rest of the layer: fp32(mu) for every row of the padded
// workspace (0 beyond M), and the rounding remainder fp32(mu - fp32(mu)) for rows < M.
__device__ __forceinline__ float write_row_mean(const LowRankParams& p, int row, double mu64) {
  const float mh = static_cast<float>(mu64);
  if (row < p.M) {
    p.mu_out[row] = mh;
    p.mulo_out[static_cast<int64_t>(row) * p.mulo_stride] = static_cast<float>(mu64 - static_cast<double>(mh));
  } else if (row < p.m_pad) {
    p.mu_out[row] = 0.f;
  }
  return mh;
}

// Cluster reduction of the S partials: the fp32 U partials ([64][128] column-major in each
// CTA's smem) and, for the statistics, the float64 row sums (psum[128]). CTA ks finalises
// rows [ks*128/S, (ks+1)*128/S); S threads per row, 64/S columns each, summed over the
// source CTAs in rank order (deterministic). Every thread of a row forms the same mean.
template <int S>
__device__ __forceinline__ void lowrank_finish(const LowRankParams& p, const float* part,
                                               const double* psum, int m0, int ks, int t) {
  constexpr int kRows = 128 / S, kCols = 64 / S;
  const int rl = ks * kRows + t % kRows;
  const int j0 = (t / kRows) * kCols;
  const int row = m0 + rl;
  float mu = 0.f;
  if (p.stats) {
    double sum = 0.0;
#pragma unroll
    for (int src = 0; src < S; ++src)
      sum += ld_shared_cluster_f64(mapa_shared(smem_u32(psum + rl), static_cast<uint32_t>(src)));
    const double mu64 = sum / static_cast<double>(p.K);
    mu = static_cast<float>(mu64);
    if (j0 == 0) write_row_mean(p, row, mu64);
  } else if (p.mu != nullptr && row < p.M) {
    mu = p.mu[row];
  }
  if (!p.lowrank) return;
  float acc[kCols];
#pragma unroll
  for (int c = 0; c < kCols; ++c) acc[c] = 0.f;
#pragma unroll
  for (int src = 0; src < S; ++src) {
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const uint32_t la = smem_u32(part + (j0 + c) * 128 + rl);
      acc[c] += ld_shared_cluster_f32(mapa_shared(la, static_cast<uint32_t>(src)));
    }
  }
  bool over = false;
  if (row < p.M) {
    const URowTerms rt = u_row_terms(p, row, mu);
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.u + static_cast<size_t>(row) * kRankPad + j0);
#pragma unroll
    for (int c = 0; c < kCols; c += 2)
      dst[c / 2] = f2_to_half2_sat(u_value(p, rt, acc[c], j0 + c), u_value(p, rt, acc[c + 1], j0 + c + 1),
                                   over);
  }
  report_u_range(p.err, over);
}

// Warps: 0 TMA producer, 1 TMEM allocator and MMA issuer, 2..5 epilogue (thread = tile row).
// With `stats` the epilogue warps also sum each staged row piece as it lands (before the
// stage is released), which gives the token means of a centred layer from the same read of
// X; with `lowrank` off only that part runs (no L1' stream, no TMEM, no MMA).
template <int NS>
__global__ void __launch_bounds__(192, 1) k_lowrank_u(const __grid_constant__ LowRankParams p) {
  using namespace lowrank;
  constexpr int kStages = NS;                          // TMA ring depth
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // no extra alignment offset: every CTA of a cluster must use the same smem offsets
  uint8_t* smem = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  uint8_t* stage0 = smem + 1024;
  float* part = reinterpret_cast<float*>(stage0);   // [64][128] after the main loop (S > 1)
  double* psum = reinterpret_cast<double*>(stage0 + kStages * kStageBytes);   // [128] (S > 1)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // After the row-staged quantizer (`reverse`) the row tiles are taken from the last to the
  // first: that kernel's band of rows moves from the first row to the last, so the rows
  // it read last are still in L2 when these CTAs start. As the first kernel of the
  // streaming path the natural order is kept (the streaming quantizer walks backwards).
  const int mt = p.reverse ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  const int ks = blockIdx.y, S = gridDim.y;
  const int m0 = mt * kTileM;
  const int KT = static_cast<int>(cdiv(p.K, kChunkK));
  const bool lr = p.lowrank != 0, stats = p.stats != 0;
  // the S CTAs of a row tile take the 64-element K chunks in turn (chunk i S + ks), so
  // that at any time they read neighbouring 128-byte pieces of the same rows
  const int nk = KT > ks ? (KT - ks + S - 1) / S : 0;
  // first kernel of a call: clear the device error word (see k_quantize_rows)
  if (p.clear_err && blockIdx.x == 0 && ks == 0 && threadIdx.x == 0 && p.err != nullptr) *p.err = 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], (lr ? 1 : 0) + (stats ? 4 : 0));   // MMA commit, epilogue warps
    }
    mbar_init(accf, 1);
    fence_mbar_init();
    prefetch_tmap(&p.tmap_x);
    if (lr) prefetch_tmap(&p.tmap_l1);
  }
  if (lr && warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = lr ? *tmem_slot : 0u;
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      bool loads_ok = true;            // every issued load was taken by its consumers
      const uint32_t bytes = lr ? kStageBytes : kABytes;
      int i = 0;
      for (; i < nk; ++i) {
        const int s = i % kStages;
        if (i >= kStages &&
            !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, p.err, KQ_DEV_ERR_TIMEOUT_EMPTY)) {
          loads_ok = false;
          break;
        }
        uint8_t* a = stage0 + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        const int kc = i * S + ks;
        tma_load_2d(a, &p.tmap_x, kc * kChunkK, m0, &full[s]);
        if (lr) tma_load_2d(a + kABytes, &p.tmap_l1, kc * kChunkK, 0, &full[s]);
      }
      if (!loads_ok) drain_ring(full, kStages, i);
    }
  } else if (warp == 1) {
    if (lr && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTileM, kUCols);
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1, p.err, KQ_DEV_ERR_TIMEOUT_FULL)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(stage0 + s * kStageBytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int kk = 0; kk < kChunkK / 16; ++kk)
          mma_bf16(tmem, sdesc_sw128_kmajor(a + 32 * kk), sdesc_sw128_kmajor(b + 32 * kk), idesc,
                   (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
  } else {
    // epilogue warps 2..5: TMEM lane quadrant = warp % 4; thread owns tile row rl
    const int q = warp & 3;
    const int rl = 32 * q + lane;
    const int row = m0 + rl;
    bool ok = true;
    double rsum = 0.0;
    if (stats) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / kStages) & 1, p.err, KQ_DEV_ERR_TIMEOUT_FULL));
        if (!ok) break;
        rsum += chunk_row_sum(stage0 + s * kStageBytes, rl);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    if (lr) ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, p.err, KQ_DEV_ERR_TIMEOUT_ACC) && ok);
    // without the statistics the token means come from the quantize grid launched just
    // before this one; every CTA also waits for the preceding grid before exiting, so the
    // GEMM's wait on this grid covers both
    grid_dep_wait();
    tc_fence_after();
    float u[64];
    if (lr) {
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t hi[32], lo[32];
        tmem_ld_32x32b_x32(tbase + 32 * h, hi);
        tmem_ld_32x32b_x32(tbase + 64 + 32 * h, lo);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) u[32 * h + j] = __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
      }
    }
    if (!ok || nk == 0 || !lr) {
#pragma unroll
      for (int j = 0; j < 64; ++j) u[j] = 0.f;
    }
    if (S == 1) {
      float mu = 0.f;
      if (stats) mu = ok ? write_row_mean(p, row, rsum / static_cast<double>(p.K)) : 0.f;
      else if (p.mu != nullptr && row < p.M) mu = p.mu[row];
      bool over = false;
      if (lr && ok && row < p.M) {
        const URowTerms rt = u_row_terms(p, row, mu);
        uint32_t packed[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          packed[j] = f2_to_half2_sat(u_value(p, rt, u[2 * j], 2 * j), u_value(p, rt, u[2 * j + 1], 2 * j + 1),
                                      over);
        uint4* dst = reinterpret_cast<uint4*>(p.u + static_cast<size_t>(row) * kRankPad);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
      report_u_range(p.err, over);
    } else if (ok) {
      // (after a wait ran out, loads may still land in the ring that `part` overlays: the
      // partials are left alone and the call reports the timeout)
      if (lr) {
#pragma unroll
        for (int j = 0; j < 64; ++j) part[j * 128 + rl] = u[j];   // column-major: conflict-free
      }
      if (stats) psum[rl] = rsum;
    }
  }
  if (S > 1) {
    __syncwarp();
    cluster_sync();                       // every partial is in place
    if (warp >= 2) {
      if (S == 2) lowrank_finish<2>(p, part, psum, m0, ks, threadIdx.x - 64);
      else if (S == 4) lowrank_finish<4>(p, part, psum, m0, ks, threadIdx.x - 64);
      else lowrank_finish<8>(p, part, psum, m0, ks, threadIdx.x - 64);
    }
    __syncwarp();
    cluster_sync();                       // no CTA leaves while others still read its smem
  }
  tc_fence_before();
  __syncthreads();
  if (lr && warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------------
// k_quantize_chunks: centring, Kronecker block transform (or none) and MXFP4 encoding on
// 128-row x 64-element pieces of X
// ----------------------------------------------------------------------------------
// The token means are formed beforehand from the same 128 x 64 pieces (k_lowrank_u with
// stats, which also produces U), so no whole token row has to be staged here: X streams
// through a ring of pieces (TMA, 128-byte swizzle, row r of a piece at byte 128 r, its
// 16-byte chunk c at c ^ (r % 8)), and a thread owns one row of a piece at a time.
//
// Work items are (row tile, pair of pieces) = 128 rows x 4 blocks, walked from the last row
// tile to the first, and CTA c takes a contiguous range of them: the CTAs that start on the
// last row tiles find the rows the statistics kernel read last still in L2 (when X is
// larger than L2, only a small share of it: ~8 % on a 215 MB activation).
// Warps: 0 TMA producer; 1..12 three groups of four consumer warps (thread = tile row),
// group g taking every third item of the CTA's range. Per item a thread centres, transforms
// and encodes its row's 4 blocks (the two blocks of each piece in one unrolled body), writes
// 64 bytes of codes and one 32-bit scale word.
namespace chunkq {
constexpr int kStages = 8;
constexpr int kGroups = 3;
constexpr int kThreads = 32 * (1 + 4 * kGroups);
constexpr uint32_t kStageBytes = 128 * 128;             // 128 rows x 64 bf16
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytes + 1024;
}  // namespace chunkq

template <int KIND, int CENTER, bool DEBUG_XT>
__global__ void __launch_bounds__(chunkq::kThreads, 1) k_quantize_chunks(const __grid_constant__ ChunkParams p) {
  using namespace chunkq;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint8_t* stage0 = smem + 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = p.K / kBlock;
  const int KC = static_cast<int>(cdiv(p.K, 64));
  const int PP = p.pairs;
  const int nb_pad = static_cast<int>(p.katoms) * 4;
  const int64_t T = static_cast<int64_t>(p.tiles) * PP;
  const int64_t G = gridDim.x;
  const int64_t q0 = T * blockIdx.x / G, q1 = T * (blockIdx.x + 1) / G;

  if (p.clear_err && blockIdx.x == 0 && threadIdx.x == 0 && p.err != nullptr) *p.err = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 4); }
    fence_mbar_init();
    prefetch_tmap(&p.tmap_x);
  }
  __syncthreads();
  grid_dep_launch();                       // the GEMM may start its prologue

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int64_t n = 0;
      bool ok = true;
      for (int64_t q = q0; q < q1 && ok; ++q) {
        const int tile = p.tiles - 1 - static_cast<int>(q / PP);
        const int pair = static_cast<int>(q % PP);
        for (int cc = 0; cc < 2; ++cc, ++n) {
          const int s = static_cast<int>(n % kStages);
          if (n >= kStages &&
              !mbar_wait(&empty[s], static_cast<uint32_t>(n / kStages - 1) & 1u, p.err,
                         KQ_DEV_ERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          const int chunk = 2 * pair + cc;
          if (chunk < KC) {
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_2d(stage0 + s * kStageBytes, &p.tmap_x, chunk * 64, tile * 128, &full[s]);
          } else {
            mbar_arrive(&full[s]);         // K % 128 == 64: the pair's second piece is empty
          }
        }
      }
      if (!ok) drain_ring(full, kStages, n);
    }
  } else {
    // ------------------------------------------------------------- consumers
    const int cw = warp - 1;
    const int g = cw >> 2;
    const int rl = 32 * (cw & 3) + lane;
    // the means come from the statistics kernel; every CTA waits for it before exiting,
    // so the GEMM's wait on this grid covers both
    grid_dep_wait();
    uint64_t Ap[16], Bp[32];
    if (KIND == 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) Ap[i] = p.Ap[i];
#pragma unroll
      for (int i = 0; i < 32; ++i) Bp[i] = p.Bp[i];
    }
    float mh = 0.f, ml = 0.f;
    // Kronecker + centring: x - mu_hi per element, and the remainder mu_lo enters the
    // transform's second stage as the constant -mu_lo (1^T P)[8k + l] = -mu_lo sA[k] sB[l]
    uint64_t bias2[16];
    auto set_bias = [&](float lo) {
      if (KIND == 1 && CENTER) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int lp = 0; lp < 4; ++lp)
            bias2[4 * k + lp] = f2pack(-lo * p.colsumA[k] * p.colsumB[2 * lp],
                                       -lo * p.colsumA[k] * p.colsumB[2 * lp + 1]);
      }
    };
    set_bias(0.f);
    int cur_tile = -1;
    if (DEBUG_XT && CENTER) {
      // one tile per CTA in the debug launch; the rounding remainders of the means sit in
      // the first element of each output row until this CTA overwrites its rows
      const int tile = p.tiles - 1 - static_cast<int>(q0 / PP);
      const int row = tile * 128 + rl;
      if (row < p.M) { mh = p.mu[row]; ml = p.mulo[static_cast<int64_t>(row) * p.mulo_stride]; }
      set_bias(ml);
      cur_tile = tile;
      asm volatile("bar.sync 1, %0;" ::"n"(32 * 4 * kGroups) : "memory");
    }
    bool ok = true;
    for (int64_t q = q0 + g; q < q1 && ok; q += kGroups) {
      const int tile = p.tiles - 1 - static_cast<int>(q / PP);
      const int pair = static_cast<int>(q % PP);
      const int row = tile * 128 + rl;
      if (CENTER && tile != cur_tile) {
        cur_tile = tile;
        mh = row < p.M ? p.mu[row] : 0.f;
        ml = row < p.M ? p.mulo[static_cast<int64_t>(row) * p.mulo_stride] : 0.f;
        set_bias(ml);
      }
      if (!CENTER && pair == 0 && p.mu_clear != nullptr) p.mu_clear[row] = 0.f;   // row < m_pad
      uint32_t sbw = 0;
      // both pieces of the item landed first, then their four blocks in one unrolled body:
      // independent transform chains for the scheduler (measured on the video-DiT layer:
      // 120.3 us one block at a time, 115.2 us per piece, 111.3 us per item)
      const int64_t n0 = 2 * (q - q0);
      const int s0 = static_cast<int>(n0 % kStages), s1 = static_cast<int>((n0 + 1) % kStages);
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&full[s0], static_cast<uint32_t>(n0 / kStages) & 1u, p.err,
                                KQ_DEV_ERR_TIMEOUT_FULL) &&
                      mbar_wait(&full[s1], static_cast<uint32_t>((n0 + 1) / kStages) & 1u, p.err,
                                KQ_DEV_ERR_TIMEOUT_FULL));
      if (!ok) break;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int s = cc ? s1 : s0;
        const uint8_t* rowp = stage0 + s * kStageBytes + static_cast<uint32_t>(rl) * 128u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int b = 4 * pair + 2 * cc + h;
          if (b >= nb) continue;
          uint64_t v2[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(
                rowp + 16u * (static_cast<uint32_t>(4 * h + c) ^ (static_cast<uint32_t>(rl) & 7u)));
            v2[4 * c + 0] = bf16x2_to_f2(w.x);
            v2[4 * c + 1] = bf16x2_to_f2(w.y);
            v2[4 * c + 2] = bf16x2_to_f2(w.z);
            v2[4 * c + 3] = bf16x2_to_f2(w.w);
          }
          if (CENTER && KIND == 1) {
            const uint64_t m2h = f2pack(mh, mh);
#pragma unroll
            for (int i = 0; i < 16; ++i) v2[i] = fsub2(v2[i], m2h);
          } else if (CENTER) {
            const uint64_t m2h = f2pack(mh, mh), m2l = f2pack(ml, ml);
#pragma unroll
            for (int i = 0; i < 16; ++i) v2[i] = fsub2(fsub2(v2[i], m2h), m2l);
          }
          if (KIND == 1 && CENTER) kron_apply2_bias(v2, Ap, Bp, bias2);
          else if (KIND == 1) kron_apply2(v2, Ap, Bp);
          if (DEBUG_XT) {
            if (row < p.M) {
              float4* o = reinterpret_cast<float4*>(p.xt + static_cast<size_t>(row) * p.K + b * kBlock);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = make_float4(f2lo(v2[2 * i]), f2hi(v2[2 * i]), f2lo(v2[2 * i + 1]), f2hi(v2[2 * i + 1]));
            }
            continue;
          }
          const uint32_t sb = mx_scale_byte(amax32_2(v2));
          uint32_t c4[4];
          encode_scaled2(v2, mx_inv_scale(sb), c4);
          if (row < p.M)
            *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * (p.K / 2) + b * 16) =
                make_uint4(c4[0], c4[1], c4[2], c4[3]);
          sbw |= sb << (8 * (2 * cc + h));
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s0]);
        mbar_arrive(&empty[s1]);
      }
      if (!DEBUG_XT && ok) {
        // scales of blocks 4 pair .. 4 pair + 3 (0 past the last block); the row's padding
        // block groups are zeroed with its last pair. Rows M .. m_pad - 1 get zero scales.
        *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, 4 * pair, p.katoms)) = sbw;
        if (pair == PP - 1)
          for (int bb = 4 * PP; bb < nb_pad; bb += 4)
            *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, bb, p.katoms)) = 0u;
      }
    }
  }
}

template <int KIND, int CENTER, bool DBG>
static cudaError_t launch_chunks_t(const ChunkParams& p, bool dependent, int num_sms, cudaStream_t st) {
  auto fn = k_quantize_chunks<KIND, CENTER, DBG>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(chunkq::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t items = static_cast<int64_t>(p.tiles) * p.pairs;
  // the debug launch gives each CTA exactly one row tile (see the remainders above)
  int64_t grid = DBG ? p.tiles : (items < num_sms ? items : num_sms);
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(chunkq::kThreads);
  cfg.dynamicSmemBytes = chunkq::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, fn, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quantize_chunks(const ChunkParams& p, int kind, bool center, bool debug_xt,
                                   bool dependent, int num_sms, cudaStream_t st) {
#define KQ_CHUNKS(KD, C)                                                               \
  if (kind == KD && center == (C != 0))                                                \
    return debug_xt ? launch_chunks_t<KD, C, true>(p, dependent, num_sms, st)          \
                    : launch_chunks_t<KD, C, false>(p, dependent, num_sms, st);
  KQ_CHUNKS(0, 0) KQ_CHUNKS(0, 1) KQ_CHUNKS(1, 0) KQ_CHUNKS(1, 1)
#undef KQ_CHUNKS
  return cudaErrorInvalidValue;
}

// ----------------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------------
template <int KIND, int CENTER, bool DBG, bool LUT = false>
static cudaError_t launch_rows_t(const QuantParams& p, int num_sms, int block, size_t smem,
                                 cudaStream_t st) {
  auto fn = k_quantize_rows<KIND, CENTER, DBG, LUT>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = cdiv(p.M, p.unit_rows);
  int64_t grid = num_sms;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  fn<<<static_cast<unsigned>(grid), block, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const QuantParams& p, bool debug_xt, int num_sms,
                                 cudaStream_t st) {
  const int block = 32 * p.consumer_warps;
  const size_t smem = p.smem_bytes;
  const int kind = p.kind, c = p.center ? (p.ln ? 2 : 1) : 0;
  // Lloyd-Max output (the debug entry stops before the encoder and takes the MXFP4 path)
  if (p.lut && !debug_xt) {
    if (kind == 0 && c == 0) return launch_rows_t<0, 0, false, true>(p, num_sms, block, smem, st);
    if (kind == 0 && c == 1) return launch_rows_t<0, 1, false, true>(p, num_sms, block, smem, st);
    if (kind == 2 && c == 0) return launch_rows_t<2, 0, false, true>(p, num_sms, block, smem, st);
    if (kind == 2 && c == 1) return launch_rows_t<2, 1, false, true>(p, num_sms, block, smem, st);
    return cudaErrorInvalidValue;
  }
#define KQ_DISPATCH(KD, C)                                                             \
  if (kind == KD && c == C)                                                            \
    return debug_xt ? launch_rows_t<KD, C, true>(p, num_sms, block, smem, st)          \
                    : launch_rows_t<KD, C, false>(p, num_sms, block, smem, st);
  KQ_DISPATCH(0, 0) KQ_DISPATCH(0, 1) KQ_DISPATCH(0, 2) KQ_DISPATCH(1, 0) KQ_DISPATCH(1, 1)
  KQ_DISPATCH(1, 2) KQ_DISPATCH(2, 0) KQ_DISPATCH(2, 1) KQ_DISPATCH(2, 2) KQ_DISPATCH(3, 0)
#undef KQ_DISPATCH
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode_f32(const float* V, int M, int K, uint8_t* codes, uint8_t* scales,
                              cudaStream_t st, double lp) {
  const int64_t n = static_cast<int64_t>(M) * (K / kBlock);
  const int block = 256;
  const int64_t grid = cdiv(n, block);
  if (n == 0) return cudaSuccess;
  k_encode_f32<<<static_cast<unsigned>(grid), block, 0, st>>>(V, M, K, codes, scales, lp);
  return cudaGetLastError();
}

cudaError_t launch_lowrank_u(const LowRankParams& p, cudaStream_t st, bool dependent) {
  using namespace lowrank;
  auto fn = p.deep ? k_lowrank_u<kStagesDeep> : k_lowrank_u<kStages>;
  const uint32_t smem = smem_bytes(p.deep ? kStagesDeep : kStages);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cdiv(p.M, kTileM)), static_cast<unsigned>(p.split));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(p.split);
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, fn, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kq
