// Canonical <-> internal layout conversions (declarations).
#pragma once
#include "kq_internal.cuh"

namespace kq {

cudaError_t pack_weights(const WeightsLayout& WL, const uint8_t* r_codes, const uint8_t* r_scales,
                         const float* L1p, const uint16_t* L2, const float* s, uint8_t* w,
                         cudaStream_t st);
cudaError_t unpack_weights(const WeightsLayout& WL, const uint8_t* w, uint8_t* r_codes,
                           uint8_t* r_scales, float* L1p, uint16_t* L2, float* c1, float* s,
                           cudaStream_t st);
cudaError_t pack_act(const ActLayout& AL, int rank, const uint8_t* codes, const uint8_t* scales,
                     const float* mu, const uint16_t* U, uint8_t* act, cudaStream_t st);
// Lloyd-Max layers: the residual decoded to fp16 [N, K] into the weights' rf16 region.
cudaError_t decode_residual_f16(const WeightsLayout& WL, uint8_t* w, cudaStream_t st);
cudaError_t unpack_act(const ActLayout& AL, int rank, const uint8_t* act, uint8_t* codes,
                       uint8_t* scales, float* mu, uint16_t* U, cudaStream_t st);

}  // namespace kq
