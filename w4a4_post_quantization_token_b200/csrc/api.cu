// C-ABI entry points of libkq (declared in include/kq.h): argument validation on the
// host, TMA descriptor creation, and kernel launches on the caller's stream.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/kq.h"
#include "kq_internal.cuh"
#include "kq_pack.cuh"
#include "kq_prepare.cuh"

using namespace kq;

namespace {

// ------------------------------------------------------------------ device checks --
struct DeviceInfo { bool ok = false; int sms = 0; int device = 0; };

kq_status current_device(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KQ_ERR_CUDA;
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  std::lock_guard<std::mutex> g(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  if (!cache[dev].ok) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return KQ_ERR_CUDA;
    if (major != 10 || minor != 0) return KQ_ERR_NO_SM100;
    cache[dev].ok = true;
    cache[dev].sms = sms;
    cache[dev].device = dev;
  }
  *out = cache[dev];
  return KQ_OK;
}

// -------------------------------------------------------------- tensor maps (TMA) --
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool encode_fn() {
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D tiled map: inner extent (elements), outer extent (rows), row pitch (bytes).
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle sw) {
  if (!encode_fn()) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- validation --------
// TMA tensor maps and bulk copies need 16-byte global addresses; every region the library
// carves out of a caller buffer starts at a 1024-byte multiple from its base
bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kRpbhMaxK = 32736;    // largest K % 32 == 0 with 2 K < 65536

kq_status check_desc(const kq_layer_desc* d) {
  if (!d) return KQ_ERR_INVALID_ARG;
  if (d->K <= 0 || d->N <= 0 || d->rank < 0) return KQ_ERR_INVALID_ARG;
  if (d->K % 32 != 0 || d->N % 16 != 0 || d->rank > kRankPad) return KQ_ERR_UNSUPPORTED_SHAPE;
  if (d->center != 0 && d->center != 1) return KQ_ERR_INVALID_ARG;
  switch (d->t.kind) {
    case KQ_T_NONE: break;
    case KQ_T_KRON:
      if (!d->t.A || !d->t.B) return KQ_ERR_INVALID_ARG;
      if (d->t.a_dim != 4 || d->t.b_dim != 8) return KQ_ERR_UNSUPPORTED_SHAPE;
      for (int i = 0; i < 16; ++i) if (!std::isfinite(d->t.A[i])) return KQ_ERR_INVALID_ARG;
      for (int i = 0; i < 64; ++i) if (!std::isfinite(d->t.B[i])) return KQ_ERR_INVALID_ARG;
      break;
    case KQ_T_RPBH: {
      if (!d->t.perm || !d->t.sign) return KQ_ERR_INVALID_ARG;
      // the gather table holds 16-bit byte offsets into a staged row: 2 K < 65536
      if (d->K > kRpbhMaxK) return KQ_ERR_UNSUPPORTED_SHAPE;
      uint64_t seen[kRpbhMaxK / 64 + 1] = {};            // on the stack: no allocation per call
      for (int k = 0; k < d->K; ++k) {
        const int32_t p = d->t.perm[k];
        if (p < 0 || p >= d->K || ((seen[p >> 6] >> (p & 63)) & 1u)) return KQ_ERR_INVALID_ARG;
        seen[p >> 6] |= 1ull << (p & 63);
        if (d->t.sign[k] != 1 && d->t.sign[k] != -1) return KQ_ERR_INVALID_ARG;
      }
      break;
    }
    default: return KQ_ERR_INVALID_ARG;
  }
  if (d->codebook != KQ_CB_MXFP4 && d->codebook != KQ_CB_LLOYDMAX) return KQ_ERR_INVALID_ARG;
  // the codebook is designed for the Gaussian coordinates of the RPBH rotation
  if (d->codebook == KQ_CB_LLOYDMAX && (d->t.kind == KQ_T_KRON || d->ln.on != 0))
    return KQ_ERR_INVALID_ARG;
  if (d->ln.on != 0) {
    // the front-end normalises, then the layer centres the normalised token (CentriQ)
    if (d->ln.on != 1 || d->center != 1) return KQ_ERR_INVALID_ARG;
    if (!(d->ln.eps > 0.f) || !std::isfinite(d->ln.eps)) return KQ_ERR_INVALID_ARG;
  }
  return KQ_OK;
}

// gamma and beta are read only where they are written into the weights
kq_status check_ln_values(const kq_layer_desc* d) {
  if (d->ln.on == 0) return KQ_OK;
  if (!d->ln.gamma || !d->ln.beta) return KQ_ERR_INVALID_ARG;
  for (int k = 0; k < d->K; ++k)
    if (!std::isfinite(d->ln.gamma[k]) || !std::isfinite(d->ln.beta[k])) return KQ_ERR_INVALID_ARG;
  return KQ_OK;
}

WeightsLayout wlayout(const kq_layer_desc* d) {
  return WeightsLayout::make(d->K, d->N, d->rank, d->center != 0, d->t.kind, d->ln.on != 0,
                             d->codebook == KQ_CB_LLOYDMAX);
}
ActLayout alayout(const kq_layer_desc* d, int M) {
  return ActLayout::make(M, d->K, d->rank, d->ln.on != 0, d->codebook == KQ_CB_LLOYDMAX);
}

// LayerNorm table image (layout: ln_table_bytes). Position j of block b holds channel
// perm[32 b + j] for RPBH (the transform gathers its input), channel 32 b + j otherwise.
void ln_table(const kq_layer_desc* d, std::vector<uint8_t>* out) {
  const int K = d->K, nb = K / kBlock;
  const bool rpbh = d->t.kind == KQ_T_RPBH;
  out->assign(ln_table_bytes(K, d->t.kind), 0);
  uint8_t* o = out->data();
  auto put = [&](size_t at, float v) { std::memcpy(o + at, &v, 4); };
  for (int b = 0; b < nb; ++b)
    for (int j = 0; j < kBlock; ++j) {
      const uint32_t c = static_cast<uint32_t>(j / 4), e = static_cast<uint32_t>(j % 4);
      const int src = rpbh ? d->t.perm[kBlock * b + j] : kBlock * b + j;
      const size_t at = static_cast<size_t>(b) * 256 + ln_chunk_off(static_cast<uint32_t>(b), c) + 4 * e;
      put(at, d->ln.gamma[src]);
      put(at + 128, d->ln.beta[src]);
      if (rpbh)
        put(static_cast<size_t>(K) * 8 + static_cast<size_t>(b) * 128 +
                ln_chunk_off(static_cast<uint32_t>(b), c) + 4 * e,
            d->ln.gamma[kBlock * b + j]);
    }
  double sb = 0.0;
  for (int k = 0; k < K; ++k) sb += static_cast<double>(d->ln.beta[k]);
  const double mean_b = sb / static_cast<double>(K);
  std::memcpy(o + out->size() - 16, &mean_b, 8);
}

// Front-end parts of the prepared weights: gamma, beta, the kernel's table and, with a
// low-rank branch, diag(gamma) L1' and gamma^T L1', beta^T L1' (from the stored L1').
kq_status write_ln_weights(const kq_layer_desc* d, uint8_t* w, cudaStream_t st) {
  if (d->ln.on == 0) return KQ_OK;
  const WeightsLayout WL = wlayout(d);
  const size_t kb = static_cast<size_t>(d->K) * 4;
  std::vector<uint8_t> tab;
  ln_table(d, &tab);
  if (cudaMemcpyAsync(w + WL.lng, d->ln.gamma, kb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(w + WL.lnb, d->ln.beta, kb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(w + WL.lntab, tab.data(), tab.size(), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return KQ_ERR_CUDA;
  if (d->rank > 0 &&
      launch_ln_fold(reinterpret_cast<const uint16_t*>(w + WL.l1t),
                     reinterpret_cast<const float*>(w + WL.lng), reinterpret_cast<const float*>(w + WL.lnb),
                     d->K, reinterpret_cast<uint16_t*>(w + WL.l1gt), reinterpret_cast<float*>(w + WL.cg),
                     reinterpret_cast<float*>(w + WL.cb), st) != cudaSuccess)
    return KQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KQ_ERR_CUDA;   // host table
  return KQ_OK;
}

// 16-level Lloyd-Max quantizer of N(0, 1): Lloyd's alternation of the two optimality
// conditions (thresholds at the midpoints of neighbouring levels; each level the mean of
// N(0, 1) over its cell, (pdf(a) - pdf(b)) / (cdf(b) - cdf(a))), in float64 from a uniform
// start, the levels kept symmetric about 0, until a sweep moves no level by more than
// 1e-15. Computed once; the 8 positive levels and the 7 thresholds between them.
struct LloydMax { double mag[8]; double thr[7]; };
const LloydMax& lloyd_max16() {
  static LloydMax lm;
  static std::once_flag once;
  std::call_once(once, [] {
    constexpr int n = 16;
    const double inv_sqrt_2pi = 0.3989422804014327;
    auto pdf = [&](double x) { return inv_sqrt_2pi * std::exp(-0.5 * x * x); };
    auto cdf = [](double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); };
    double lv[n], nx[n];
    for (int i = 0; i < n; ++i) lv[i] = -2.0 + 4.0 * i / (n - 1);
    for (int it = 0; it < 200000; ++it) {
      double move = 0.0;
      for (int i = 0; i < n; ++i) {
        const bool lo_inf = i == 0, hi_inf = i == n - 1;
        const double a = lo_inf ? 0.0 : 0.5 * (lv[i - 1] + lv[i]);
        const double b = hi_inf ? 0.0 : 0.5 * (lv[i] + lv[i + 1]);
        const double pa = lo_inf ? 0.0 : pdf(a), pb = hi_inf ? 0.0 : pdf(b);
        const double ca = lo_inf ? 0.0 : cdf(a), cb = hi_inf ? 1.0 : cdf(b);
        nx[i] = (pa - pb) / (cb - ca);
      }
      for (int i = 0; i < n / 2; ++i) {
        const double v = 0.5 * (nx[n - 1 - i] - nx[i]);
        nx[i] = -v;
        nx[n - 1 - i] = v;
      }
      for (int i = 0; i < n; ++i) {
        move = std::fmax(move, std::fabs(nx[i] - lv[i]));
        lv[i] = nx[i];
      }
      if (move < 1e-15) break;
    }
    for (int i = 0; i < 8; ++i) lm.mag[i] = lv[8 + i];
    for (int i = 0; i < 7; ++i) lm.thr[i] = 0.5 * (lm.mag[i] + lm.mag[i + 1]);
  });
  return lm;
}

// Gauss-Jordan inverse with partial pivoting (float64); false if singular.
bool invert(const double* a, int n, double* inv) {
  std::vector<double> m(static_cast<size_t>(n) * 2 * n, 0.0);
  for (int i = 0; i < n; ++i) {
    for (int j = 0; j < n; ++j) m[i * 2 * n + j] = a[i * n + j];
    m[i * 2 * n + n + i] = 1.0;
  }
  double scale = 0.0;
  for (int i = 0; i < n * n; ++i) scale = std::fmax(scale, std::fabs(a[i]));
  if (scale == 0.0) return false;
  for (int c = 0; c < n; ++c) {
    int piv = c;
    for (int r = c + 1; r < n; ++r)
      if (std::fabs(m[r * 2 * n + c]) > std::fabs(m[piv * 2 * n + c])) piv = r;
    if (std::fabs(m[piv * 2 * n + c]) <= 1e-12 * scale) return false;
    if (piv != c)
      for (int j = 0; j < 2 * n; ++j) std::swap(m[c * 2 * n + j], m[piv * 2 * n + j]);
    const double p = m[c * 2 * n + c];
    for (int j = 0; j < 2 * n; ++j) m[c * 2 * n + j] /= p;
    for (int r = 0; r < n; ++r) {
      if (r == c) continue;
      const double f = m[r * 2 * n + c];
      if (f != 0.0)
        for (int j = 0; j < 2 * n; ++j) m[r * 2 * n + j] -= f * m[c * 2 * n + j];
    }
  }
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) inv[i * n + j] = m[i * 2 * n + n + j];
  return true;
}

// 32x32 Kronecker block (row-major): (A (x) B)[8i + j][8k + l] = A[i][k] B[j][l]
void kron32(const double* A, const double* B, double* P) {
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 8; ++j)
      for (int k = 0; k < 4; ++k)
        for (int l = 0; l < 8; ++l) P[(8 * i + j) * 32 + 8 * k + l] = A[4 * i + k] * B[8 * j + l];
}

// RPBH tables as stored in the weights buffer: int32 perm, float sign/sqrt(32)
void rpbh_tables(const kq_layer_desc* d, std::vector<float>* sgn) {
  sgn->resize(static_cast<size_t>(d->K));
  const float rs = static_cast<float>(1.0 / std::sqrt(32.0));
  for (int k = 0; k < d->K; ++k) (*sgn)[k] = d->t.sign[k] < 0 ? -rs : rs;
}

// The RPBH table image the quantize kernel copies into shared memory (layout.cuh).
void rpbh_qtab(const kq_layer_desc* d, std::vector<uint8_t>* out) {
  const int K = d->K, nb = K / kBlock;
  out->assign(qtab_bytes(K), 0);
  uint16_t* pt = reinterpret_cast<uint16_t*>(out->data());
  for (int k = 0; k < K; ++k)
    pt[swz64(static_cast<uint32_t>(k) * 2u) / 2] =
        static_cast<uint16_t>(swz64(static_cast<uint32_t>(d->t.perm[k]) * 2u));
  uint32_t* sm = reinterpret_cast<uint32_t*>(out->data() + static_cast<size_t>(K) * 2);
  for (int b = 0; b < nb; ++b)
    for (int w = 0; w < 4; ++w) {
      uint32_t m = 0;
      for (int j = 0; j < 8; ++j) m |= (d->t.sign[32 * b + 8 * w + j] < 0 ? 8u : 0u) << (4 * j);
      sm[4 * b + w] = m;
    }
}

// Shape of the quantize kernel's work: rows per unit, warps and slots per warp.
// A unit's u * K/32 blocks should fill the warp's lanes (>= 85% busy); among the shapes
// whose slots fit in shared memory take the most warps, then two slots per warp (the
// next unit loads while this one is computed) over one.
struct QuantShape { int u = 0, warps = 0, stages = 0; };
QuantShape choose_quant_shape(int K, size_t slot_avail, int max_warps) {
  const int nb = K / kBlock;
  const size_t rstride = align_up(static_cast<size_t>(K) * 2, 512);
  int u_eff = 32;
  for (int u = 1; u <= 32; ++u) {
    const int iters = (u * nb + 31) / 32;
    if (static_cast<double>(u * nb) >= 0.85 * 32.0 * iters) { u_eff = u; break; }
  }
  QuantShape q;
  for (int warps = max_warps; warps >= 1; warps -= (warps > 4 ? 4 : 1))
    for (int stages = 2; stages >= 1; --stages)
      for (int u = u_eff; u >= 1; --u)
        if (static_cast<size_t>(warps) * stages * u * rstride <= slot_avail) {
          if (q.warps == 0 || (u == u_eff && q.u != u_eff)) { q.u = u; q.warps = warps; q.stages = stages; }
          if (u == u_eff) return q;
          break;
        }
  return q;
}

// inv_s non-null selects the SmoothQuant comparator (kind 3): per-channel multiply by
// inv_s instead of the layer's block transform (the layer must have none).
kq_status fill_quant_params(const kq_layer_desc* d, const void* weights, const void* X, int M,
                            uint8_t* act, QuantParams* p, const DeviceInfo& di,
                            const float* inv_s = nullptr) {
  std::memset(p, 0, sizeof(*p));
  const WeightsLayout WL = wlayout(d);
  const ActLayout AL = alayout(d, M);
  const int K = d->K, nb = K / kBlock;
  if (d->t.kind == KQ_T_KRON) {
    auto pair = [](float lo, float hi) {
      uint32_t a, b;
      std::memcpy(&a, &lo, 4);
      std::memcpy(&b, &hi, 4);
      return (static_cast<uint64_t>(b) << 32) | a;
    };
    for (int i = 0; i < 4; ++i)
      for (int k = 0; k < 4; ++k) p->Ap[4 * i + k] = pair(d->t.A[4 * i + k], d->t.A[4 * i + k]);
    for (int j = 0; j < 8; ++j)
      for (int l = 0; l < 4; ++l) p->Bp[4 * j + l] = pair(d->t.B[8 * j + 2 * l], d->t.B[8 * j + 2 * l + 1]);
  }
  p->M = M; p->K = K; p->m_pad = static_cast<int>(AL.m_pad);
  p->kind = inv_s ? 3 : d->t.kind; p->center = d->center;
  p->inv_s = inv_s;
  p->katoms = sf_katoms(K);
  // each row is staged in a 512-byte aligned slot row (its own 64-byte swizzle pattern),
  // loaded in boxes of up to 256 lines
  const uint32_t rstride = static_cast<uint32_t>(align_up(static_cast<size_t>(K) * 2, 512));
  int box = 1;
  for (int c = 1; c <= 256 && c <= nb; ++c) if (nb % c == 0) box = c;
  p->box_lines = box;
  p->row_stride = rstride;
  if (!make_tmap(&p->tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 32,
                 static_cast<uint64_t>(M) * nb, 64, 32, static_cast<uint32_t>(box),
                 CU_TENSOR_MAP_SWIZZLE_64B))
    return KQ_ERR_CUDA;
  const bool ln = d->ln.on != 0;
  const bool lut = d->codebook == KQ_CB_LLOYDMAX;
  if ((ln || lut) && inv_s) return KQ_ERR_INVALID_ARG;
  p->tables_off = (ln || lut) ? kQTablesMinLn : kQTablesMin;
  if (lut) {
    const LloydMax& cb = lloyd_max16();
    p->lut = 1;
    for (int i = 0; i < 8; ++i) p->lut_mag[i] = static_cast<float>(cb.mag[i]);
    for (int i = 0; i < 7; ++i) p->lut_thr[i] = static_cast<float>(cb.thr[i]);
  }
  p->qtab_bytes = d->t.kind == KQ_T_RPBH ? static_cast<uint32_t>(qtab_bytes(K)) : 0u;
  const size_t table_bytes = inv_s ? static_cast<size_t>(K) * 4 : p->qtab_bytes;
  size_t tables_end = p->tables_off + table_bytes;
  if (ln) {
    p->ln = 1;
    p->ln_eps = static_cast<double>(d->ln.eps);
    p->lntab_off = static_cast<uint32_t>(align_up(tables_end, 128));
    p->lntab_bytes = static_cast<uint32_t>(ln_table_bytes(K, d->t.kind));
    tables_end = p->lntab_off + p->lntab_bytes;
  }
  p->bufs_off = align_up(tables_end, 1024);
  constexpr size_t kSmemMax = 227 * 1024;
  if (p->bufs_off + rstride > kSmemMax) return KQ_ERR_UNSUPPORTED_SHAPE;
  const int max_warps = d->t.kind == KQ_T_KRON ? kQMaxWarpsKron : kQMaxWarps;
  QuantShape q = choose_quant_shape(K, kSmemMax - p->bufs_off, max_warps);
  if (q.warps == 0) return KQ_ERR_UNSUPPORTED_SHAPE;
  // With a low-rank branch, prefer an 8-warp footprint whose shared memory leaves room for
  // one k_lowrank_u CTA on the same SM (that kernel is a programmatic dependent and reads
  // the token means only in its epilogue). The low-rank kernel's 255 registers keep the
  // two apart all the same (192 x 255 + 256 x 106 exceed the 64 K register file); a
  // 164-register low-rank epilogue that let them share measured no faster. Not for the
  // Kronecker transform: that kernel is FMA-bound and 16 warps win (measured: video layer
  // 314 -> 295 us).
  if (d->rank > 0 && d->t.kind != KQ_T_KRON) {
    const size_t share = kSmemPerSM - 2 * kSmemPerBlockReserved - kLowRankSmemBytes;
    if (p->bufs_off + rstride <= share) {
      const QuantShape q2 = choose_quant_shape(K, share - p->bufs_off, max_warps < 8 ? max_warps : 8);
      if (q2.warps == 8) q = q2;
    }
  }
  p->unit_rows = q.u;
  p->consumer_warps = q.warps;
  p->nbufs = q.stages;
  p->smem_bytes = p->bufs_off + static_cast<size_t>(q.warps) * q.stages * q.u * rstride;
  (void)di;
  if (act) {
    p->codes = act + AL.codes;
    p->sf = act + AL.sf;
    p->mu = reinterpret_cast<float*>(act + AL.mu);
    p->err = reinterpret_cast<uint32_t*>(act + AL.err);
    if (ln) {
      p->lnm = reinterpret_cast<float*>(act + AL.lnm);
      p->lnr = reinterpret_cast<float*>(act + AL.lnr);
    }
    if (lut) {
      p->a16 = reinterpret_cast<uint16_t*>(act + AL.codes);
      p->sig = reinterpret_cast<float*>(act + AL.sig);
      p->codes = nullptr;
      p->sf = nullptr;
    }
  }
  p->qtab = weights ? static_cast<const uint8_t*>(weights) + WL.qtab : nullptr;
  if (ln) p->lntab = weights ? static_cast<const uint8_t*>(weights) + WL.lntab : nullptr;
  return KQ_OK;
}

// Layers whose transform is Kronecker or none, without the LayerNorm front-end or the
// codebook, take the streaming path: k_lowrank_u forms U and (centring) the token means from
// 128-row x 64-element pieces of X, then k_quantize_chunks centres, transforms and encodes
// the same pieces. The other layers (RPBH's global gather, the front-end's statistics, the
// codebook's sigma) stage whole token rows in k_quantize_rows.
bool chunk_path(const kq_layer_desc* d) {
  return (d->t.kind == KQ_T_KRON || d->t.kind == KQ_T_NONE) && d->ln.on == 0 &&
         d->codebook == KQ_CB_MXFP4;
}

void kron_pairs(const kq_layer_desc* d, uint64_t* Ap, uint64_t* Bp) {
  auto pair = [](float lo, float hi) {
    uint32_t a, b;
    std::memcpy(&a, &lo, 4);
    std::memcpy(&b, &hi, 4);
    return (static_cast<uint64_t>(b) << 32) | a;
  };
  for (int i = 0; i < 4; ++i)
    for (int k = 0; k < 4; ++k) Ap[4 * i + k] = pair(d->t.A[4 * i + k], d->t.A[4 * i + k]);
  for (int j = 0; j < 8; ++j)
    for (int l = 0; l < 4; ++l) Bp[4 * j + l] = pair(d->t.B[8 * j + 2 * l], d->t.B[8 * j + 2 * l + 1]);
}

// The streaming path. act == nullptr is the debug launch: Xt [M, K] and mu [M] are written
// instead of the workspace (the means' rounding remainders are parked in Xt[row][0] until
// the quantize kernel overwrites that row).
kq_status run_chunk_path(const kq_layer_desc* d, const void* weights, const void* X, int M,
                         uint8_t* act, float* xt, float* mu_dbg, cudaStream_t st,
                         const DeviceInfo& di, bool keep_err) {
  const WeightsLayout WL = wlayout(d);
  const ActLayout AL = alayout(d, M);
  const bool debug = act == nullptr;
  const bool center = d->center != 0;
  const bool lr = d->rank > 0 && !debug;
  const int K = d->K;
  ChunkParams cp;
  std::memset(&cp, 0, sizeof(cp));
  if (!make_tmap(&cp.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K),
                 static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return KQ_ERR_CUDA;
  if (d->t.kind == KQ_T_KRON) {
    kron_pairs(d, cp.Ap, cp.Bp);
    for (int k = 0; k < 4; ++k) {
      double a = 0.0;
      for (int i = 0; i < 4; ++i) a += d->t.A[4 * i + k];
      cp.colsumA[k] = static_cast<float>(a);
    }
    for (int l = 0; l < 8; ++l) {
      double b = 0.0;
      for (int j = 0; j < 8; ++j) b += d->t.B[8 * j + l];
      cp.colsumB[l] = static_cast<float>(b);
    }
  }
  cp.M = M; cp.K = K;
  cp.m_pad = static_cast<int>(AL.m_pad);
  cp.tiles = static_cast<int>(cdiv(M, 128));
  cp.pairs = static_cast<int>(cdiv(K, 128));
  cp.katoms = sf_katoms(K);
  uint32_t* err = debug ? nullptr : reinterpret_cast<uint32_t*>(act + AL.err);
  float* mu = debug ? mu_dbg : reinterpret_cast<float*>(act + AL.mu);
  float* mulo = debug ? xt : reinterpret_cast<float*>(act + AL.mulo);
  const int64_t mulo_stride = debug ? K : 1;
  bool first = true;
  if (center || lr) {
    LowRankParams lp;
    std::memset(&lp, 0, sizeof(lp));
    lp.tmap_x = cp.tmap_x;
    if (lr) {
      const uint8_t* w = static_cast<const uint8_t*>(weights);
      if (!make_tmap(&lp.tmap_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w + WL.l1t, static_cast<uint64_t>(K),
                     kUCols, static_cast<uint64_t>(K) * 2, 64, kUCols, CU_TENSOR_MAP_SWIZZLE_128B))
        return KQ_ERR_CUDA;
      lp.c1 = reinterpret_cast<const float*>(w + WL.c1);
      lp.u = reinterpret_cast<uint16_t*>(act + AL.u);
    }
    lp.lowrank = lr ? 1 : 0;
    lp.stats = center ? 1 : 0;
    lp.clear_err = (!debug && !keep_err) ? 1 : 0;
    lp.m_pad = debug ? M : static_cast<int>(AL.m_pad);
    lp.mu_out = mu;
    lp.mulo_out = mulo;
    lp.mulo_stride = mulo_stride;
    lp.M = M; lp.K = K; lp.split = u_split(M, K);
    lp.deep = 1;                         // alone on its SMs: the deep ring
    lp.err = err;
    if (launch_lowrank_u(lp, st, /*dependent=*/false) != cudaSuccess) return KQ_ERR_CUDA;
    first = false;
  } else if (debug) {
    if (cudaMemsetAsync(mu_dbg, 0, static_cast<size_t>(M) * 4, st) != cudaSuccess) return KQ_ERR_CUDA;
  }
  cp.clear_err = (first && !debug && !keep_err) ? 1 : 0;
  cp.mu = center ? mu : nullptr;
  cp.mulo = center ? mulo : nullptr;
  cp.mulo_stride = mulo_stride;
  cp.mu_clear = (center || debug) ? nullptr : reinterpret_cast<float*>(act + AL.mu);
  cp.codes = debug ? nullptr : act + AL.codes;
  cp.sf = debug ? nullptr : act + AL.sf;
  cp.xt = debug ? xt : nullptr;
  cp.err = err;
  if (launch_quantize_chunks(cp, d->t.kind == KQ_T_KRON ? 1 : 0, center, debug, !first, di.sms, st) !=
      cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status run_quantize(const kq_layer_desc* d, const void* weights, const void* X, int M,
                       uint8_t* act, cudaStream_t st, const DeviceInfo& di, bool keep_err = false) {
  if (chunk_path(d)) return run_chunk_path(d, weights, X, M, act, nullptr, nullptr, st, di, keep_err);
  const WeightsLayout WL = wlayout(d);
  const ActLayout AL = alayout(d, M);
  QuantParams qp;
  kq_status s = fill_quant_params(d, weights, X, M, act, &qp, di);
  if (s != KQ_OK) return s;
  qp.keep_err = keep_err ? 1 : 0;
  if (launch_quantize_rows(qp, false, di.sms, st) != cudaSuccess) return KQ_ERR_CUDA;
  if (d->rank > 0) {
    LowRankParams lp;
    std::memset(&lp, 0, sizeof(lp));
    if (!make_tmap(&lp.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(d->K),
                   static_cast<uint64_t>(M), static_cast<uint64_t>(d->K) * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
    const bool ln = d->ln.on != 0;
    const uint8_t* w = static_cast<const uint8_t*>(weights);
    if (!make_tmap(&lp.tmap_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w + (ln ? WL.l1gt : WL.l1t),
                   static_cast<uint64_t>(d->K), kUCols, static_cast<uint64_t>(d->K) * 2, 64, kUCols,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
    lp.c1 = reinterpret_cast<const float*>(w + WL.c1);
    if (ln) {
      lp.ln = 1;
      lp.cg = reinterpret_cast<const float*>(w + WL.cg);
      lp.cb = reinterpret_cast<const float*>(w + WL.cb);
      lp.lnm = reinterpret_cast<const float*>(act + AL.lnm);
      lp.lnr = reinterpret_cast<const float*>(act + AL.lnr);
    }
    lp.lowrank = 1;
    lp.stats = 0;                        // the means come from the quantize kernel
    lp.reverse = 1;                      // the quantize kernel's last rows are in L2
    lp.mu = d->center ? reinterpret_cast<const float*>(act + AL.mu) : nullptr;
    lp.u = reinterpret_cast<uint16_t*>(act + AL.u);
    lp.M = M; lp.K = d->K; lp.split = u_split(M, d->K);
    // 3-stage ring when the quantize shape left shared memory for a low-rank CTA beside it,
    // else the deep ring
    lp.deep = qp.smem_bytes + kLowRankSmemBytes + 2 * kSmemPerBlockReserved > kSmemPerSM ? 1 : 0;
    lp.err = reinterpret_cast<uint32_t*>(act + AL.err);
    if (launch_lowrank_u(lp, st) != cudaSuccess) return KQ_ERR_CUDA;
  }
  return KQ_OK;
}

kq_status run_gemm(const kq_layer_desc* d, const void* weights, const uint8_t* act, int M, void* Y,
                   int out_dtype, cudaStream_t st, const DeviceInfo& di) {
  const WeightsLayout WL = wlayout(d);
  const ActLayout AL = alayout(d, M);
  const uint8_t* w = static_cast<const uint8_t*>(weights);
  const int K = d->K, N = d->N;
  const uint32_t bn = static_cast<uint32_t>(gemm_tile_n());
  const bool bf16 = out_dtype == KQ_OUT_BF16;
  GemmParams gp;
  std::memset(&gp, 0, sizeof(gp));
  if (d->codebook == KQ_CB_LLOYDMAX) {
    // fp16 operand [M, K] and fp16 residual [N, K], 64-element (128-byte) k-tiles
    gp.f16 = 1;
    if (!make_tmap(&gp.tmap_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, act + AL.codes, static_cast<uint64_t>(K),
                   static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
    if (!make_tmap(&gp.tmap_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w + WL.rf16, static_cast<uint64_t>(K),
                   static_cast<uint64_t>(N), static_cast<uint64_t>(K) * 2, 64, bn,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
  } else {
    if (!make_tmap(&gp.tmap_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, act + AL.codes, static_cast<uint64_t>(K / 2),
                   static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), 128, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
    if (!make_tmap(&gp.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w + WL.rcodes, static_cast<uint64_t>(K / 2),
                   static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), 128, bn,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return KQ_ERR_CUDA;
  }
  // low-rank step: only the first 32 of the 64 stored columns when rank <= 32 (the rest
  // are zero), as 64-byte rows with the 64-byte swizzle
  const int lrk = d->rank == 0 ? 0 : (d->rank <= 32 ? 32 : kRankPad);
  if (d->rank > 0) {
    const CUtensorMapSwizzle sw = lrk == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_tmap(&gp.tmap_u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, act + AL.u, kRankPad,
                   static_cast<uint64_t>(M), kRankPad * 2, static_cast<uint32_t>(lrk), 128, sw))
      return KQ_ERR_CUDA;
    if (!make_tmap(&gp.tmap_l2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w + WL.l2t, kRankPad,
                   static_cast<uint64_t>(N), kRankPad * 2, static_cast<uint32_t>(lrk), bn, sw))
      return KQ_ERR_CUDA;
  }
  if (!make_tmap(&gp.tmap_y, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                 Y, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(N) * (bf16 ? 2 : 4), bf16 ? 64 : 32, 32,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return KQ_ERR_CUDA;
  gp.sfa = act + AL.sf;
  gp.sfb = w + WL.rsf;
  gp.mu = d->center ? reinterpret_cast<const float*>(act + AL.mu) : nullptr;
  gp.s = reinterpret_cast<const float*>(w + WL.s);
  gp.y = Y;
  gp.M = M; gp.N = N; gp.K = K;
  gp.rank_pad = lrk;
  gp.katoms = sf_katoms(K);
  gp.err = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(act) + AL.err);
  if (launch_gemm(gp, bf16, di.sms, st) != cudaSuccess) return KQ_ERR_CUDA;
  return KQ_OK;
}

}  // namespace

// =====================================================================================
namespace {

kq_status prepare_weights_impl(const kq_layer_desc* desc, const void* W_bf16, void* weights, void* ws,
                               size_t ws_bytes, kq_stream_t stream, double lp) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if ((s = check_ln_values(desc)) != KQ_OK) return s;
  if (!W_bf16 || !weights || !ws) return KQ_ERR_INVALID_ARG;
  if (!aligned(W_bf16) || !aligned(weights) || !aligned(ws)) return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  const size_t lw = prepare_syevd_lwork(desc->K, desc->N, desc->rank);
  if (lw == 0) return KQ_ERR_CUDA;
  if (ws_bytes < PrepareWs::make(desc->K, desc->N, desc->rank, lw).total)
    return KQ_ERR_WORKSPACE_TOO_SMALL;

  double pinv[32 * 32], pfwd[32 * 32];
  for (int i = 0; i < 32 * 32; ++i) pinv[i] = pfwd[i] = (i / 32 == i % 32) ? 1.0 : 0.0;
  if (desc->t.kind == KQ_T_KRON) {
    double A[16], B[64], Ai[16], Bi[64];
    for (int i = 0; i < 16; ++i) A[i] = desc->t.A[i];
    for (int i = 0; i < 64; ++i) B[i] = desc->t.B[i];
    if (!invert(A, 4, Ai) || !invert(B, 8, Bi)) return KQ_ERR_SINGULAR_TRANSFORM;
    kron32(Ai, Bi, pinv);
    kron32(A, B, pfwd);
  }
  std::vector<float> sgn;
  if (desc->t.kind == KQ_T_RPBH) rpbh_tables(desc, &sgn);

  PrepareArgs a;
  a.K = desc->K; a.N = desc->N; a.rank = desc->rank; a.kind = desc->t.kind;
  a.center = desc->center != 0;
  a.W = W_bf16; a.weights = weights; a.ws = ws; a.syevd_lwork = lw;
  a.pinv_host = pinv; a.pfwd_host = pfwd;
  a.perm_host = desc->t.kind == KQ_T_RPBH ? desc->t.perm : nullptr;
  a.sgn_host = desc->t.kind == KQ_T_RPBH ? sgn.data() : nullptr;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.lp = lp;
  if (run_prepare(a) != PrepStatus::Ok) return KQ_ERR_CUDA;
  if (desc->t.kind == KQ_T_RPBH) {
    std::vector<uint8_t> qtab;
    rpbh_qtab(desc, &qtab);
    if (cudaMemcpyAsync(static_cast<uint8_t*>(weights) + wlayout(desc).qtab, qtab.data(), qtab.size(),
                        cudaMemcpyHostToDevice, a.stream) != cudaSuccess ||
        cudaStreamSynchronize(a.stream) != cudaSuccess)
      return KQ_ERR_CUDA;
  }
  if (desc->codebook == KQ_CB_LLOYDMAX &&
      (decode_residual_f16(wlayout(desc), static_cast<uint8_t*>(weights), a.stream) != cudaSuccess ||
       cudaStreamSynchronize(a.stream) != cudaSuccess))
    return KQ_ERR_CUDA;
  return write_ln_weights(desc, static_cast<uint8_t*>(weights), a.stream);
}

// Streams and events of the host-buffer entry, one set per device, created on first use.
// The copies of one call run on two streams of their own (host-to-device, device-to-
// host) so that they overlap each other and the kernels; kq_linear_host orders them
// against the caller's stream with events.
constexpr int kHostChunksMax = 8;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t ev_in[kHostChunksMax] = {}, ev_c[kHostChunksMax] = {};
  std::mutex mu;
  bool ok = false;
};
HostPipe* host_pipe(int device) {
  static std::mutex m;
  static HostPipe* pipes[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> g(m);
  if (!pipes[device]) {
    HostPipe* h = new HostPipe;
    bool ok = cudaStreamCreateWithFlags(&h->in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kHostChunksMax; ++i)
      ok = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->ev_c[i], cudaEventDisableTiming) == cudaSuccess;
    h->ok = ok;
    pipes[device] = h;
  }
  return pipes[device]->ok ? pipes[device] : nullptr;
}

// kq_linear's device work with the device error word kept (row chunks after the first)
kq_status linear_dev(const kq_layer_desc* desc, const void* weights, const void* X, int32_t M,
                     void* Y, int32_t out_dtype, void* act, size_t act_bytes, cudaStream_t st,
                     const DeviceInfo& di, bool keep_err) {
  if (M <= 0 || !weights || !X || !act || !Y) return KQ_ERR_INVALID_ARG;
  if (!aligned(weights) || !aligned(X) || !aligned(act) || !aligned(Y)) return KQ_ERR_ALIGNMENT;
  if (act_bytes < alayout(desc, M).total) return KQ_ERR_WORKSPACE_TOO_SMALL;
  kq_status s = run_quantize(desc, weights, X, M, static_cast<uint8_t*>(act), st, di, keep_err);
  if (s != KQ_OK) return s;
  return run_gemm(desc, weights, static_cast<const uint8_t*>(act), M, Y, out_dtype, st, di);
}

}  // namespace

extern "C" {

const char* kq_status_string(kq_status s) {
  switch (s) {
    case KQ_OK: return "ok";
    case KQ_ERR_INVALID_ARG: return "invalid argument";
    case KQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case KQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case KQ_ERR_SINGULAR_TRANSFORM: return "Kronecker factor is singular";
    case KQ_ERR_WORKSPACE_TOO_SMALL: return "buffer smaller than the size query";
    case KQ_ERR_CUDA: return "CUDA call failed";
    case KQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case KQ_ERR_NO_SM100: return "device is not sm_100 (B200)";
    case KQ_ERR_LOWRANK_RANGE: return "a low-rank activation exceeded the fp16 range (saturated)";
  }
  return "unknown status";
}

kq_status kq_lloydmax_codebook(double* levels8, double* thresholds7) {
  const LloydMax& cb = lloyd_max16();
  if (levels8) for (int i = 0; i < 8; ++i) levels8[i] = cb.mag[i];
  if (thresholds7) for (int i = 0; i < 7; ++i) thresholds7[i] = cb.thr[i];
  return KQ_OK;
}

const char* kq_version(void) { return "kq 0.1 (sm_100a, tcgen05 mxf4)"; }

size_t kq_weights_bytes(const kq_layer_desc* desc) {
  if (check_desc(desc) != KQ_OK) return 0;
  return wlayout(desc).total;
}

size_t kq_act_bytes(const kq_layer_desc* desc, int32_t M) {
  if (check_desc(desc) != KQ_OK || M <= 0) return 0;
  return alayout(desc, M).total;
}

size_t kq_prepare_ws_bytes(const kq_layer_desc* desc) {
  if (check_desc(desc) != KQ_OK) return 0;
  const size_t lw = prepare_syevd_lwork(desc->K, desc->N, desc->rank);
  if (lw == 0) return 0;
  return PrepareWs::make(desc->K, desc->N, desc->rank, lw).total;
}

kq_status kq_prepare_weights(const kq_layer_desc* desc, const void* W_bf16, void* weights, void* ws,
                             size_t ws_bytes, kq_stream_t stream) {
  return prepare_weights_impl(desc, W_bf16, weights, ws, ws_bytes, stream, 0.0);
}

kq_status kq_prepare_weights_lp(const kq_layer_desc* desc, double p, const void* W_bf16,
                                void* weights, void* ws, size_t ws_bytes, kq_stream_t stream) {
  if (!(p > 0.0 && p <= 2.0)) return KQ_ERR_INVALID_ARG;
  return prepare_weights_impl(desc, W_bf16, weights, ws, ws_bytes, stream, p);
}

kq_status kq_quantize_act(const kq_layer_desc* desc, const void* weights, const void* X_bf16,
                          int32_t M, void* act, size_t act_bytes, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (M <= 0 || !weights || !X_bf16 || !act) return KQ_ERR_INVALID_ARG;
  if (!aligned(weights) || !aligned(X_bf16) || !aligned(act)) return KQ_ERR_ALIGNMENT;
  if (act_bytes < alayout(desc, M).total) return KQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the quantize kernel's first thread clears the device error word (no separate memset
  // node in front of it)
  return run_quantize(desc, weights, X_bf16, M, static_cast<uint8_t*>(act), st, di);
}

kq_status kq_smooth_quantize_act(const kq_layer_desc* desc, const float* inv_s,
                                 const void* X_bf16, int32_t M, void* act, size_t act_bytes,
                                 kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (desc->t.kind != KQ_T_NONE || desc->center || desc->rank != 0 || desc->ln.on ||
      desc->codebook != KQ_CB_MXFP4)
    return KQ_ERR_INVALID_ARG;
  if (M <= 0 || !inv_s || !X_bf16 || !act) return KQ_ERR_INVALID_ARG;
  if (!aligned(inv_s) || !aligned(X_bf16) || !aligned(act)) return KQ_ERR_ALIGNMENT;
  if (act_bytes < alayout(desc, M).total) return KQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* a = static_cast<uint8_t*>(act);
  QuantParams qp;
  if ((s = fill_quant_params(desc, nullptr, X_bf16, M, a, &qp, di, inv_s)) != KQ_OK) return s;
  if (launch_quantize_rows(qp, false, di.sms, st) != cudaSuccess) return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_gemm(const kq_layer_desc* desc, const void* weights, const void* act, int32_t M,
                  void* Y, int32_t out_dtype, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (M <= 0 || !weights || !act || !Y) return KQ_ERR_INVALID_ARG;
  if (out_dtype != KQ_OUT_F32 && out_dtype != KQ_OUT_BF16) return KQ_ERR_INVALID_ARG;
  if (!aligned(weights) || !aligned(act) || !aligned(Y)) return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  return run_gemm(desc, weights, static_cast<const uint8_t*>(act), M, Y, out_dtype,
                  reinterpret_cast<cudaStream_t>(stream), di);
}

kq_status kq_linear(const kq_layer_desc* desc, const void* weights, const void* X_bf16, int32_t M,
                    void* Y, int32_t out_dtype, void* act, size_t act_bytes, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!Y) return KQ_ERR_INVALID_ARG;
  if (out_dtype != KQ_OUT_F32 && out_dtype != KQ_OUT_BF16) return KQ_ERR_INVALID_ARG;
  if (!aligned(Y)) return KQ_ERR_ALIGNMENT;
  s = kq_quantize_act(desc, weights, X_bf16, M, act, act_bytes, stream);
  if (s != KQ_OK) return s;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  return run_gemm(desc, weights, static_cast<const uint8_t*>(act), M, Y, out_dtype,
                  reinterpret_cast<cudaStream_t>(stream), di);
}

kq_status kq_linear_host(const kq_layer_desc* desc, const void* weights, const void* X_host,
                         void* X_dev, int32_t M, void* Y_host, void* Y_dev, int32_t out_dtype,
                         void* act, size_t act_bytes, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!X_host || !Y_host || !X_dev || !Y_dev || M <= 0) return KQ_ERR_INVALID_ARG;
  if (out_dtype != KQ_OUT_F32 && out_dtype != KQ_OUT_BF16) return KQ_ERR_INVALID_ARG;
  if (!weights || !act) return KQ_ERR_INVALID_ARG;
  if (!aligned(weights) || !aligned(X_dev) || !aligned(Y_dev) || !aligned(act)) return KQ_ERR_ALIGNMENT;
  if (act_bytes < alayout(desc, M).total) return KQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t xrow = static_cast<size_t>(desc->K) * 2;
  const size_t yrow = static_cast<size_t>(desc->N) * (out_dtype == KQ_OUT_BF16 ? 2 : 4);
  // Rows in chunks of a 128 multiple (>= 512 rows, <= 8 chunks): the copy-in of chunk
  // i + 1, the kernels of chunk i and the copy-out of chunk i - 1 run at the same time
  // (PCIe moves both directions at once). One chunk: everything on `stream`.
  int nch = M >= 1024 ? std::min(kHostChunksMax, M / 512) : 1;
  const int C = static_cast<int>(align_up(static_cast<size_t>(cdiv(M, nch)), 128));
  nch = static_cast<int>(cdiv(M, C));
  HostPipe* hp = nch > 1 ? host_pipe(di.device) : nullptr;
  if (!hp) {
    if (cudaMemcpyAsync(X_dev, X_host, M * xrow, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return KQ_ERR_CUDA;
    if ((s = linear_dev(desc, weights, X_dev, M, Y_dev, out_dtype, act, act_bytes, st, di, false)) != KQ_OK)
      return s;
    if (cudaMemcpyAsync(Y_host, Y_dev, M * yrow, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return KQ_ERR_CUDA;
    return KQ_OK;
  }
  std::lock_guard<std::mutex> g(hp->mu);
  if (cudaEventRecord(hp->start, st) != cudaSuccess || cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return KQ_ERR_CUDA;
  for (int i = 0; i < nch && s == KQ_OK; ++i) {
    const size_t r0 = static_cast<size_t>(i) * C;
    const int rows = static_cast<int>(std::min<size_t>(C, M - r0));
    if (cudaMemcpyAsync(static_cast<uint8_t*>(X_dev) + r0 * xrow, static_cast<const uint8_t*>(X_host) + r0 * xrow,
                        rows * xrow, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
        cudaEventRecord(hp->ev_in[i], hp->in) != cudaSuccess || cudaStreamWaitEvent(st, hp->ev_in[i], 0) != cudaSuccess) {
      s = KQ_ERR_CUDA;
      break;
    }
    if ((s = linear_dev(desc, weights, static_cast<uint8_t*>(X_dev) + r0 * xrow, rows,
                        static_cast<uint8_t*>(Y_dev) + r0 * yrow, out_dtype, act, act_bytes, st, di,
                        i > 0)) != KQ_OK)
      break;
    if (cudaEventRecord(hp->ev_c[i], st) != cudaSuccess || cudaStreamWaitEvent(hp->out, hp->ev_c[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(Y_host) + r0 * yrow, static_cast<const uint8_t*>(Y_dev) + r0 * yrow,
                        rows * yrow, cudaMemcpyDeviceToHost, hp->out) != cudaSuccess)
      s = KQ_ERR_CUDA;
  }
  // whatever was enqueued, the caller's stream is ordered after both copy streams
  if (cudaEventRecord(hp->ev_c[0], hp->in) != cudaSuccess || cudaStreamWaitEvent(st, hp->ev_c[0], 0) != cudaSuccess ||
      cudaEventRecord(hp->done, hp->out) != cudaSuccess || cudaStreamWaitEvent(st, hp->done, 0) != cudaSuccess)
    return KQ_ERR_CUDA;
  return s;
}

kq_status kq_weights_pack(const kq_layer_desc* desc, const void* r_codes, const void* r_scales,
                          const float* L1p_f32, const void* L2_bf16, const float* s_col,
                          void* weights, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!r_codes || !r_scales || !s_col || !weights) return KQ_ERR_INVALID_ARG;
  if (desc->rank > 0 && (!L1p_f32 || !L2_bf16)) return KQ_ERR_INVALID_ARG;
  if ((s = check_ln_values(desc)) != KQ_OK) return s;
  if (!aligned(weights)) return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  const WeightsLayout WL = wlayout(desc);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(weights);
  if (pack_weights(WL, static_cast<const uint8_t*>(r_codes), static_cast<const uint8_t*>(r_scales),
                   L1p_f32, static_cast<const uint16_t*>(L2_bf16), s_col, w, st) != cudaSuccess)
    return KQ_ERR_CUDA;
  if (desc->t.kind == KQ_T_RPBH) {
    std::vector<float> sgn;
    std::vector<uint8_t> qtab;
    rpbh_tables(desc, &sgn);
    rpbh_qtab(desc, &qtab);
    if (cudaMemcpyAsync(w + WL.perm, desc->t.perm, static_cast<size_t>(desc->K) * 4,
                        cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(w + WL.sgn, sgn.data(), static_cast<size_t>(desc->K) * 4,
                        cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(w + WL.qtab, qtab.data(), qtab.size(), cudaMemcpyHostToDevice, st) !=
            cudaSuccess)
      return KQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KQ_ERR_CUDA;   // host locals
  }
  if (desc->codebook == KQ_CB_LLOYDMAX && decode_residual_f16(WL, w, st) != cudaSuccess)
    return KQ_ERR_CUDA;
  return write_ln_weights(desc, w, st);
}

kq_status kq_weights_unpack(const kq_layer_desc* desc, const void* weights, void* r_codes,
                            void* r_scales, float* L1p_f32, void* L2_bf16, float* c1, float* s_col,
                            kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!weights) return KQ_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  if (unpack_weights(wlayout(desc), static_cast<const uint8_t*>(weights),
                     static_cast<uint8_t*>(r_codes), static_cast<uint8_t*>(r_scales), L1p_f32,
                     static_cast<uint16_t*>(L2_bf16), c1, s_col,
                     reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_act_pack(const kq_layer_desc* desc, const void* codes, const void* scales,
                      const float* mu, const void* U_bf16, int32_t M, void* act, size_t act_bytes,
                      kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (M <= 0 || !codes || !scales || !act) return KQ_ERR_INVALID_ARG;
  if (desc->center && !mu) return KQ_ERR_INVALID_ARG;
  if (desc->rank > 0 && !U_bf16) return KQ_ERR_INVALID_ARG;
  if (!aligned(act)) return KQ_ERR_ALIGNMENT;
  if (act_bytes < alayout(desc, M).total) return KQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  if (pack_act(alayout(desc, M), desc->rank, static_cast<const uint8_t*>(codes),
               static_cast<const uint8_t*>(scales), mu, static_cast<const uint16_t*>(U_bf16),
               static_cast<uint8_t*>(act), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_act_unpack(const kq_layer_desc* desc, const void* act, int32_t M, void* codes,
                        void* scales, float* mu, void* U_bf16, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (M <= 0 || !act) return KQ_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  if (unpack_act(alayout(desc, M), desc->rank, static_cast<const uint8_t*>(act),
                 static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), mu,
                 static_cast<uint16_t*>(U_bf16), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_debug_transform(const kq_layer_desc* desc, const void* weights, const void* X_bf16,
                             int32_t M, float* Xt, float* mu, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (M <= 0 || !weights || !X_bf16 || !Xt || !mu) return KQ_ERR_INVALID_ARG;
  if (!aligned(X_bf16) || !aligned(Xt) || !aligned(weights)) return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  if (chunk_path(desc))
    return run_chunk_path(desc, weights, X_bf16, M, nullptr, Xt, mu, reinterpret_cast<cudaStream_t>(stream),
                          di, false);
  QuantParams qp;
  s = fill_quant_params(desc, weights, X_bf16, M, nullptr, &qp, di);
  if (s != KQ_OK) return s;
  // m_pad = M: no padding rows in debug mode; outputs go to the caller's arrays
  qp.m_pad = M;
  qp.codes = nullptr;
  qp.sf = nullptr;
  qp.mu = mu;
  qp.xt = Xt;
  qp.err = nullptr;
  if (launch_quantize_rows(qp, true, di.sms, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_debug_encode_f32(const float* V, int32_t M, int32_t K, void* codes, void* scales,
                              kq_stream_t stream) {
  if (!V || !codes || !scales || M <= 0 || K <= 0) return KQ_ERR_INVALID_ARG;
  if (K % 32 != 0) return KQ_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(V) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u))
    return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  kq_status s = current_device(&di);
  if (s != KQ_OK) return s;
  if (launch_encode_f32(V, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_debug_encode_lp_f32(const float* V, int32_t M, int32_t K, double p, void* codes,
                                 void* scales, kq_stream_t stream) {
  if (!V || !codes || !scales || M <= 0 || K <= 0 || !(p > 0.0 && p <= 2.0)) return KQ_ERR_INVALID_ARG;
  if (K % 32 != 0) return KQ_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(V) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u))
    return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  kq_status s = current_device(&di);
  if (s != KQ_OK) return s;
  if (launch_encode_f32(V, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                        reinterpret_cast<cudaStream_t>(stream), p) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

kq_status kq_last_device_error(const kq_layer_desc* desc, void* act, int32_t M, kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!act || M <= 0) return KQ_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return KQ_ERR_CUDA;
  uint32_t word = 0;
  const ActLayout AL = alayout(desc, M);
  uint8_t* a = static_cast<uint8_t*>(act);
  if (cudaMemcpy(&word, a + AL.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return KQ_ERR_CUDA;
  if (word != 0 && cudaMemset(a + AL.err, 0, 4) != cudaSuccess) return KQ_ERR_CUDA;
  if (word & KQ_DEV_ERR_TIMEOUT_MASK) return KQ_ERR_DEVICE_TIMEOUT;
  if (word & KQ_DEV_ERR_U_RANGE) return KQ_ERR_LOWRANK_RANGE;
  return word ? KQ_ERR_DEVICE_TIMEOUT : KQ_OK;
}

kq_status kq_debug_wait_timeout(const kq_layer_desc* desc, void* act, int32_t M, uint32_t limit_us,
                                kq_stream_t stream) {
  kq_status s = check_desc(desc);
  if (s != KQ_OK) return s;
  if (!act || M <= 0 || limit_us == 0 || limit_us > 1000000u) return KQ_ERR_INVALID_ARG;
  if (!aligned(act)) return KQ_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((s = current_device(&di)) != KQ_OK) return s;
  uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(act) + alayout(desc, M).err);
  if (launch_wait_never(err, static_cast<uint64_t>(limit_us) * 1000u,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KQ_ERR_CUDA;
  return KQ_OK;
}

}  // extern "C"
