// Per-token FP8 (E4M3) quantisation of an activation tensor, scale and cast
// in one pass over memory (SparkDiffusion summary, robotworld.top, section
// 2.3: activations of the linear projections quantised to E4M3 with a
// per-token scale chosen at run time, in one fused kernel).
//
// A token's row is its H*d channels of the [B, L, H, d] bf16 tensor. Per row:
// amax = max |x|, codes = E4M3(x * (448 / amax)) rounded to nearest even and
// saturated at +-448 (cvt.rn.satfinite), scale = amax / 448, both quotients
// IEEE float32; a row of zeros gets scale 1 and zero codes.
//
// One warp per row, the whole row held in registers (16-byte loads, 8 bf16
// per lane per step), so HBM sees one read of x and one write of the codes.
// |x| of a bf16 is its bit pattern with the sign cleared, and those patterns
// order like the magnitudes, so amax is an integer max (two 16-bit lanes per
// instruction) and a warp max.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kQuantWarps = 8;

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  // the first source lands in the upper byte, the second in the lower byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int MAXC>
__global__ void __launch_bounds__(kQuantWarps * 32)
quant_fp8_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ xq, float* __restrict__ scale, long long rows,
                 int n8) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kQuantWarps + warp;
  if (row >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x) + row * n8;
  uint4 v[MAXC];
  uint32_t m2 = 0u;  // two 16-bit magnitudes
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = 32 * i + lane;
    v[i] = c < n8 ? __ldcs(src + c) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    m2 = __vmaxu2(m2, v[i].x & 0x7fff7fffu);
    m2 = __vmaxu2(m2, v[i].y & 0x7fff7fffu);
    m2 = __vmaxu2(m2, v[i].z & 0x7fff7fffu);
    m2 = __vmaxu2(m2, v[i].w & 0x7fff7fffu);
  }
  uint32_t m = max(m2 & 0xffffu, m2 >> 16);
  m = __reduce_max_sync(0xffffffffu, m);
  const float amax = __uint_as_float(m << 16);
  const bool zero = amax == 0.f;
  const float inv = zero ? 0.f : 448.f / amax;
  if (lane == 0) scale[row] = zero ? 1.f : amax / 448.f;
  uint2* dst = reinterpret_cast<uint2*>(xq) + row * n8;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = 32 * i + lane;
    if (c < n8) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t out[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint16_t a = e4m3x2(bf16_lo_f(w[2 * k]) * inv, bf16_hi_f(w[2 * k]) * inv);
        const uint16_t b = e4m3x2(bf16_lo_f(w[2 * k + 1]) * inv, bf16_hi_f(w[2 * k + 1]) * inv);
        out[k] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
      }
      __stcs(dst + c, make_uint2(out[0], out[1]));
    }
  }
}

template <int MAXC>
cudaError_t run_quant(const uint16_t* x, uint8_t* xq, float* scale, long long rows, int n8, cudaStream_t stream) {
  const long long ctas = (rows + kQuantWarps - 1) / kQuantWarps;
  quant_fp8_kernel<MAXC><<<static_cast<unsigned>(ctas), kQuantWarps * 32, 0, stream>>>(x, xq, scale, rows, n8);
  return cudaGetLastError();
}

}  // namespace

int quant_fp8_max_row() { return 64 * 32 * 8; }

cudaError_t launch_quant_fp8(const Problem& P, const uint16_t* x, uint8_t* xq, float* scale, cudaStream_t stream) {
  const long long rows = static_cast<long long>(P.B) * P.L;
  const int n8 = P.H * P.d / 8;  // 16-byte pieces per row
  const int per_lane = (n8 + 31) / 32;
  if (per_lane <= 1) return run_quant<1>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 2) return run_quant<2>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 4) return run_quant<4>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 8) return run_quant<8>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 12) return run_quant<12>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 16) return run_quant<16>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 20) return run_quant<20>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 24) return run_quant<24>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 32) return run_quant<32>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 48) return run_quant<48>(x, xq, scale, rows, n8, stream);
  if (per_lane <= 64) return run_quant<64>(x, xq, scale, rows, n8, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sda
