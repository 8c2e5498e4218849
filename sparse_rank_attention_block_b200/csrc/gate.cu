// Gate fusion (SparkDiffusion summary, robotworld.top, section 2.1, last
// equation): O_i = O_s,i + g_i r_i O_lr,i with r_i the RMS over d of O_s,i.
//
// Pure streaming kernel (reads O_s, O_lr, g; writes O): D/8 threads own one
// (token, head) row with one 16-byte load per operand, r_i is a shuffle
// reduction over those lanes, and the grid is a multiple of the SM count.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

template <int D>
__global__ void __launch_bounds__(256)
gate_kernel(Problem P, size_t rows, const uint16_t* __restrict__ o_s, const uint16_t* __restrict__ o_lr,
            const float* __restrict__ g, uint16_t* __restrict__ o) {
  constexpr int LPR = D / 8;                 // lanes per row
  constexpr int RPW = 32 / LPR;              // rows per warp
  const int lane = threadIdx.x % 32;
  const int sub = lane % LPR;
  const size_t warp_global = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const size_t warps = static_cast<size_t>(gridDim.x) * blockDim.x / 32;
  for (size_t base = warp_global * RPW; base < rows; base += warps * RPW) {
    const size_t row = base + lane / LPR;
    const bool ok = row < rows;
    uint4 xs = make_uint4(0, 0, 0, 0), xl = make_uint4(0, 0, 0, 0);
    float gv = 0.f;
    if (ok) {
      xs = __ldg(reinterpret_cast<const uint4*>(o_s + row * D) + sub);
      xl = __ldg(reinterpret_cast<const uint4*>(o_lr + row * D) + sub);
      gv = __ldg(g + (P.gate_per_head ? row : row / P.H));
    }
    const float s[8] = {bf16_lo(xs.x), bf16_hi(xs.x), bf16_lo(xs.y), bf16_hi(xs.y),
                        bf16_lo(xs.z), bf16_hi(xs.z), bf16_lo(xs.w), bf16_hi(xs.w)};
    const float lr[8] = {bf16_lo(xl.x), bf16_hi(xl.x), bf16_lo(xl.y), bf16_hi(xl.y),
                         bf16_lo(xl.z), bf16_hi(xl.z), bf16_lo(xl.w), bf16_hi(xl.w)};
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += s[e] * s[e];
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float gr = gv * sqrtf(ss / D);
    if (ok) {
      uint4 out;
      out.x = pack_bf16(fmaf(gr, lr[0], s[0]), fmaf(gr, lr[1], s[1]));
      out.y = pack_bf16(fmaf(gr, lr[2], s[2]), fmaf(gr, lr[3], s[3]));
      out.z = pack_bf16(fmaf(gr, lr[4], s[4]), fmaf(gr, lr[5], s[5]));
      out.w = pack_bf16(fmaf(gr, lr[6], s[6]), fmaf(gr, lr[7], s[7]));
      reinterpret_cast<uint4*>(o + row * D)[sub] = out;
    }
  }
}

}  // namespace

cudaError_t launch_gate_fuse(const Problem& P, const uint16_t* o_s, const uint16_t* o_lr, const float* g,
                             uint16_t* o, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t rows = static_cast<size_t>(P.B) * P.L * P.H;
  const int blocks = sms * 8;  // 8 x 256 threads per SM: full occupancy, grid-stride
  if (P.d == 128)
    gate_kernel<128><<<blocks, 256, 0, stream>>>(P, rows, o_s, o_lr, g, o);
  else
    gate_kernel<64><<<blocks, 256, 0, stream>>>(P, rows, o_s, o_lr, g, o);
  return cudaGetLastError();
}

}  // namespace sda
