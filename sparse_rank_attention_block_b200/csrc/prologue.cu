// Prologue of the path: backbone Q/K RMSNorm and full-d 3D RoPE in one pass
// (SparkDiffusion summary, robotworld.top, section 2.1: the low-rank branch
// reuses the backbone's normalised query/key; H3 portability report, section
// 2.1: the fused QKV-RoPE operator in front of the attention).
//
// Per (token, head) row of d channels, for q and for k:
//   x_norm = x / sqrt(mean_c x_c^2 + eps) * w      (w: learned weight [H, d])
//   x_rot  = RoPE_d(p) x_norm                      (all d/2 adjacent pairs)
// both written as bf16 (round to nearest even from the same fp32 x_norm).
// The d/2 pairs split over the (t, h, w) axes as (d/8, 3d/16, 3d/16); pair mu
// of an axis with n pairs turns by coordinate * base^(-mu / n).
//
// HBM-bound (read q, k; write four tensors). Every CTA first builds the
// cos/sin table of all (axis coordinate, pair) in shared memory in double
// precision; then each warp walks rows: a row is d/8 lanes of 8 channels
// (one 16-byte load per tensor), two rows per warp at d = 128, and a warp
// keeps U row groups in flight.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kProThreads = 256;
constexpr int kProUnroll = 4;   // row groups per warp in flight
constexpr int kProMaxTab = 8192;  // table entries held in shared memory (64 KB)

struct ProPairs {
  int pt, ph, pw;       // pairs per axis
  int nt, nh;           // table offsets of the h and w parts
};

__host__ __device__ inline ProPairs pro_pairs(const Problem& P) {
  ProPairs s;
  s.pt = P.d / 8;
  s.ph = 3 * P.d / 16;
  s.pw = 3 * P.d / 16;
  s.nt = P.grid_t * s.pt;
  s.nh = P.grid_h * s.ph;
  return s;
}

__host__ __device__ inline int pro_table_entries(const Problem& P) {
  const ProPairs s = pro_pairs(P);
  return s.nt + s.nh + P.grid_w * s.pw;
}

__device__ __forceinline__ float bflo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bfhi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int D>
__global__ void __launch_bounds__(kProThreads)
qk_prologue_kernel(Problem P, const uint16_t* __restrict__ q_raw, const uint16_t* __restrict__ k_raw,
                   const uint16_t* __restrict__ w_q, const uint16_t* __restrict__ w_k, uint16_t* __restrict__ q_norm,
                   uint16_t* __restrict__ k_norm, uint16_t* __restrict__ q_rot, uint16_t* __restrict__ k_rot) {
  extern __shared__ float2 tab[];
  constexpr int LPR = D / 8;         // lanes per row
  constexpr int RPW = 32 / LPR;      // rows per warp instruction
  const ProPairs pp = pro_pairs(P);
  const int n_tab = pro_table_entries(P);
  for (int e = threadIdx.x; e < n_tab; e += blockDim.x) {
    int coord, mu, n;
    if (e < pp.nt) {
      coord = e / pp.pt; mu = e % pp.pt; n = pp.pt;
    } else if (e < pp.nt + pp.nh) {
      coord = (e - pp.nt) / pp.ph; mu = (e - pp.nt) % pp.ph; n = pp.ph;
    } else {
      coord = (e - pp.nt - pp.nh) / pp.pw; mu = (e - pp.nt - pp.nh) % pp.pw; n = pp.pw;
    }
    const double theta = pow(static_cast<double>(P.rope_base), -static_cast<double>(mu) / n);
    double s, c;
    sincos(static_cast<double>(coord) * theta, &s, &c);
    tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int sub = lane / LPR;            // row of this lane within the warp's group
  const int part = lane % LPR;           // 8-channel part of the row
  const int c0 = 8 * part;               // first channel; pairs c0/2 .. c0/2 + 3
  const long long rows = static_cast<long long>(P.B) * P.L * P.H;
  const long long groups = (rows + RPW - 1) / RPW;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  const float eps = P.rms_eps;
  for (long long g0 = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + warp; g0 < groups;
       g0 += stride * kProUnroll) {
    uint4 qv[kProUnroll], kv[kProUnroll];
    long long rw[kProUnroll];
#pragma unroll
    for (int u = 0; u < kProUnroll; ++u) {
      const long long g = g0 + u * stride;
      rw[u] = g * RPW + sub;
      const bool ok = g < groups && rw[u] < rows;
      qv[u] = ok ? __ldcs(reinterpret_cast<const uint4*>(q_raw + rw[u] * D + c0)) : make_uint4(0, 0, 0, 0);
      kv[u] = ok ? __ldcs(reinterpret_cast<const uint4*>(k_raw + rw[u] * D + c0)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kProUnroll; ++u) {
      const long long r = rw[u];
      const bool ok = g0 + u * stride < groups && r < rows;
      const int h = static_cast<int>(r % P.H);
      const int l = static_cast<int>((r / P.H) % P.L);
      const int gw = l % P.grid_w, gh = (l / P.grid_w) % P.grid_h, gt = l / (P.grid_w * P.grid_h);
      const uint4 wq4 = __ldg(reinterpret_cast<const uint4*>(w_q + h * D + c0));
      const uint4 wk4 = __ldg(reinterpret_cast<const uint4*>(w_k + h * D + c0));
      const uint32_t qw[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
      const uint32_t kw[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      const uint32_t wqw[4] = {wq4.x, wq4.y, wq4.z, wq4.w};
      const uint32_t wkw[4] = {wk4.x, wk4.y, wk4.z, wk4.w};
      float sq = 0.f, sk = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sq += bflo(qw[i]) * bflo(qw[i]) + bfhi(qw[i]) * bfhi(qw[i]);
        sk += bflo(kw[i]) * bflo(kw[i]) + bfhi(kw[i]) * bfhi(kw[i]);
      }
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
      }
      const float iq = rsqrtf(sq / D + eps), ik = rsqrtf(sk / D + eps);
      uint32_t qn[4], kn[4], qr[4], kr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = c0 / 2 + i;  // pair (2m, 2m+1) = the two halves of word i
        int e;
        if (m < pp.pt) e = gt * pp.pt + m;
        else if (m < pp.pt + pp.ph) e = pp.nt + gh * pp.ph + (m - pp.pt);
        else e = pp.nt + pp.nh + gw * pp.pw + (m - pp.pt - pp.ph);
        const float2 cs = tab[e];
        const float q0 = bflo(qw[i]) * iq * bflo(wqw[i]), q1 = bfhi(qw[i]) * iq * bfhi(wqw[i]);
        const float k0 = bflo(kw[i]) * ik * bflo(wkw[i]), k1 = bfhi(kw[i]) * ik * bfhi(wkw[i]);
        qn[i] = pack_bf16(q0, q1);
        kn[i] = pack_bf16(k0, k1);
        qr[i] = pack_bf16(q0 * cs.x - q1 * cs.y, q0 * cs.y + q1 * cs.x);
        kr[i] = pack_bf16(k0 * cs.x - k1 * cs.y, k0 * cs.y + k1 * cs.x);
      }
      if (ok) {
        __stcs(reinterpret_cast<uint4*>(q_norm + r * D + c0), make_uint4(qn[0], qn[1], qn[2], qn[3]));
        __stcs(reinterpret_cast<uint4*>(k_norm + r * D + c0), make_uint4(kn[0], kn[1], kn[2], kn[3]));
        __stcs(reinterpret_cast<uint4*>(q_rot + r * D + c0), make_uint4(qr[0], qr[1], qr[2], qr[3]));
        __stcs(reinterpret_cast<uint4*>(k_rot + r * D + c0), make_uint4(kr[0], kr[1], kr[2], kr[3]));
      }
    }
  }
}

template <int D>
cudaError_t run_prologue(const Problem& P, const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* w_q,
                         const uint16_t* w_k, uint16_t* q_norm, uint16_t* k_norm, uint16_t* q_rot, uint16_t* k_rot,
                         cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(pro_table_entries(P)) * sizeof(float2);
  cudaError_t e =
      cudaFuncSetAttribute(qk_prologue_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qk_prologue_kernel<D>, kProThreads, smem);
  if (e != cudaSuccess) return e;
  // one resident wave: every CTA strides over an equal share of the rows
  const int grid = (per_sm > 0 ? per_sm : 1) * sms;
  qk_prologue_kernel<D><<<grid, kProThreads, smem, stream>>>(P, q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot);
  return cudaGetLastError();
}

}  // namespace

bool qk_prologue_supported(const Problem& P) { return pro_table_entries(P) <= kProMaxTab; }

cudaError_t launch_qk_prologue(const Problem& P, const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* w_q,
                               const uint16_t* w_k, uint16_t* q_norm, uint16_t* k_norm, uint16_t* q_rot,
                               uint16_t* k_rot, cudaStream_t stream) {
  if (P.d == 128) return run_prologue<128>(P, q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot, stream);
  if (P.d == 64) return run_prologue<64>(P, q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sda
