// fp8_cast_kernels.cuh -- the cast step before the GEMM: BF16 values to e4m3 codes with
// fine-grained fp32 scales, in the layouts the GEMM kernels read.
//
// The pages leave this step to the user (turtlesai.it summary: casting to FP8 and the transposed,
// TMA-aligned LHS scales are done outside the GEMM library; news article: fine-grained scaling).
// Per block -- 1 x 128 of a row of A, or 128 x 128 of B --
//   scale = amax / top in fp32 (1 for an all-zero block), one IEEE division, top = 448 (e4m3)
//           or 57344 (e5m2), the target format's largest finite value;
//   code  = round-to-nearest-even of the fp32 quotient x / scale in the target format,
//           saturating at +-top.
// Both kernels are bound by HBM: per element 2 bytes read and 1 byte written, plus one fp32
// scale per 128 (rows) or 16384 (blocks) elements.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace fg {

__device__ __forceinline__ void unpack_bf16x8(const uint4& raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Codes of x / s for 8 values of one block: the IEEE quotient (one correctly rounded fp32
// division per value, as the definition states), then e4m3 round-to-nearest-even with saturation.
// (A reciprocal-multiply fast path with an exact fallback near e4m3 midpoints measured slower.)
// FMT 0: e4m3 (largest finite 448), 1: e5m2 (largest finite 57344).
template <int FMT>
__device__ __forceinline__ uint2 encode_fp8x8(const float (&f)[8], float scale) {
  constexpr __nv_fp8_interpretation_t kind = FMT == 0 ? __NV_E4M3 : __NV_E5M2;
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)  // x.x goes to the low byte, i.e. the lower address
    h[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(f[2 * i], scale), __fdiv_rn(f[2 * i + 1], scale)), __NV_SATFINITE, kind));
  uint2 out;
  out.x = h[0] | (h[1] << 16);
  out.y = h[2] | (h[3] << 16);
  return out;
}

template <int FMT>
__device__ __forceinline__ float cast_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, FMT == 0 ? 448.0f : 57344.0f);
}

// A side.  X: bf16 [G*M][K] (row r = g*M + m), Q: e4m3 codes in the same layout, sfa:
// [G][ceil(K/128)][ld], element (g, kb, m) at (g*KB + kb)*ld + m.  K % 8 == 0.
// A warp takes one row and a chunk of four 256-column spans (1024 columns) per step; in each span
// lanes 0-15 hold its first K block and lanes 16-31 its second, 8 consecutive elements per lane
// (16-byte loads, all four issued before any arithmetic; 8-byte stores).
constexpr int kCastSpans = 4;
template <int FMT>
__global__ void __launch_bounds__(256) fp8_cast_rows_kernel(const __nv_bfloat16* __restrict__ X,
                                                            uint8_t* __restrict__ Q, float* __restrict__ sfa,
                                                            int M, int K, int ld, long long rows, int chunks) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int KB = (K + 127) / 128;
  for (long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < rows * chunks;
       w += nwarps) {
    const long long r = w / chunks;
    const int c = static_cast<int>(w - r * chunks);
    const __nv_bfloat16* xr = X + r * K;
    uint4 raw[kCastSpans];
#pragma unroll
    for (int j = 0; j < kCastSpans; ++j) {
      const int k = (c * kCastSpans + j) * 256 + lane * 8;
      raw[j] = k < K ? __ldg(reinterpret_cast<const uint4*>(xr + k)) : make_uint4(0u, 0u, 0u, 0u);
    }
    long long g = -1;
    int m = 0;
#pragma unroll
    for (int j = 0; j < kCastSpans; ++j) {
      if ((c * kCastSpans + j) * 256 >= K) break;  // the row ends before this span (warp-uniform)
      const int k = (c * kCastSpans + j) * 256 + lane * 8;
      float f[8];
      unpack_bf16x8(raw[j], f);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));  // half-warp
      const float scale = cast_scale<FMT>(amax);
      if (k < K) {
        *reinterpret_cast<uint2*>(Q + r * K + k) = encode_fp8x8<FMT>(f, scale);
        if ((lane & 15) == 0) {
          if (g < 0) { g = r / M; m = static_cast<int>(r - g * M); }
          sfa[(g * KB + k / 128) * ld + m] = scale;
        }
      }
    }
  }
}

// B side.  X: bf16 [G][N][K], Q: codes, sfb: [G][ceil(N/128)][ceil(K/128)].  One CTA per 128 x 128
// block (grid KB x NB x G): thread t holds rows t/16 + 16 i (i < 8) x columns 8 (t%16) .. +7 of
// the block in registers, so the block is read once.  K % 8 == 0.
template <int FMT>
__global__ void __launch_bounds__(256) fp8_cast_blocks_kernel(const __nv_bfloat16* __restrict__ X,
                                                              uint8_t* __restrict__ Q, float* __restrict__ sfb,
                                                              int N, int K) {
  __shared__ float s_max[8];
  const int kb = blockIdx.x, nb = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x;
  const int k = kb * 128 + (t & 15) * 8;
  const size_t base = static_cast<size_t>(g) * N * K;
  float f[8][8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb * 128 + (t >> 4) + 16 * i;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (n < N && k < K) raw = __ldg(reinterpret_cast<const uint4*>(X + base + static_cast<size_t>(n) * K + k));
    unpack_bf16x8(raw, f[i]);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[i][j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) s_max[t >> 5] = amax;
  __syncthreads();
  amax = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_max[w]);
  const float scale = cast_scale<FMT>(amax);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb * 128 + (t >> 4) + 16 * i;
    if (n < N && k < K)
      *reinterpret_cast<uint2*>(Q + base + static_cast<size_t>(n) * K + k) = encode_fp8x8<FMT>(f[i], scale);
  }
  if (t == 0) sfb[(static_cast<size_t>(g) * gridDim.y + nb) * gridDim.x + kb] = scale;
}

}  // namespace fg
