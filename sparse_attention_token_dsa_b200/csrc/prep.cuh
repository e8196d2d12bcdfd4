// prep.cuh — operand preparation for the FP8 indexer path.
//
// "PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 2.3 "from formula to FP8
// cache": the indexer key is stored as FP8 data plus a scale, k^ = round(k/a),
// and the dot products accumulate in higher precision before the head weights
// and the head sum.  Reading used here: one scale per row (a key row, or all
// heads of a query token), a = amax / 448 (448 = largest finite E4M3), codes by
// round-to-nearest-even with saturation; both divisions in IEEE fp32.
#pragma once
#include "common.cuh"

namespace dsa {

__device__ __forceinline__ float load_as_f32(const void* x, int dtype, int64_t i) {
  if (dtype == DSA_F32) return reinterpret_cast<const float*>(x)[i];
  return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(x)[i] << 16);
}

__device__ __forceinline__ uint8_t e4m3_rn_sat(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}

// One warp per row: amax, scale, codes.
__global__ void quantize_rows_kernel(const void* __restrict__ x, int dtype, int64_t rows,
                                     int cols, uint8_t* __restrict__ out,
                                     float* __restrict__ out_scale) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t base = row * cols;
  float amax = 0.f;
  for (int c = lane; c < cols; c += 32) amax = fmaxf(amax, fabsf(load_as_f32(x, dtype, base + c)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float a = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (lane == 0) out_scale[row] = a;
  for (int c = lane; c < cols; c += 32) out[base + c] = e4m3_rn_sat(__fdiv_rn(load_as_f32(x, dtype, base + c), a));
}

// Split of a bf16 / fp32 query head into two e4m3 parts for the e4m3-key MMA:
//   s = amax(q_j) / 448,  hi = e4m3(q_j / s),  lo = e4m3(q_j / s - hi),
//   q_j ~= s * (hi + lo).
// The residual of a round-to-nearest e4m3 code is at most half its spacing and
// is itself coded with e4m3's four significant bits (its subnormal steps of
// 2^-9 below 2^-6), so the pair carries about eight significant bits, the
// precision of the bf16 input.  As hi + lo is a plain sum, the scan runs the
// two parts as two MMAs into one accumulator.  Output layout [2][rows][H][d]
// (every row's hi part, then every row's lo part) and the scale s per
// (row, head), which the scan folds into the head weight.
__global__ void split_query_kernel(const void* __restrict__ q, int dtype, int64_t rows, int H,
                                   int d, uint8_t* __restrict__ parts,
                                   float* __restrict__ head_scale) {
  const int64_t rh = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (rh >= rows * H) return;
  const int64_t src = rh * d;
  float amax = 0.f;
  for (int c = lane; c < d; c += 32) amax = fmaxf(amax, fabsf(load_as_f32(q, dtype, src + c)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (lane == 0) head_scale[rh] = s;
  uint8_t* hi = parts + rh * (int64_t)d;
  uint8_t* lo = parts + (rows * H + rh) * (int64_t)d;
  for (int c = lane; c < d; c += 32) {
    const float v = __fdiv_rn(load_as_f32(q, dtype, src + c), s);
    const uint8_t ch = e4m3_rn_sat(v);
    hi[c] = ch;
    lo[c] = e4m3_rn_sat(v - e4m3_value(ch));
  }
}

}  // namespace dsa
