// Block selector: mean-pool Q/K per block, score pooled pairs, keep the top-k
// key blocks of every (batch, head, query block), ties to the lower index.
//
// The sparse branch A_M keeps a 1 - s fraction of query-key blocks picked by
// block-level scoring / top-k (SparkDiffusion summary, robotworld.top,
// section 2.1); the pooled-mean dot product is the scoring rule used here.
//
// Kernel 1 (pool): HBM-bound streaming read of Q and K. One CTA per
// (batch, block) covers all H heads of a contiguous [block, H*d] slab; every
// thread owns 8 consecutive channels (one 16-byte load per token) and sums its
// tokens in order, so the fp32 result does not depend on scheduling.
//
// Kernel 2 (score + select): one CTA per (batch, head, 16 query blocks).
// Scores of the 16 rows against all key blocks are built in shared memory
// (fp32 FMA in a fixed channel order), then each warp radix-selects the k-th
// largest score of its row (4 passes of 8 bits over an order-preserving
// uint32 key) and compacts the winners in ascending index order with ballots.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kPoolMaxThreads = 640;
constexpr int kRows = 16;        // query blocks per CTA in the score kernel
constexpr int kKeyChunk = 128;   // key blocks staged per pass
constexpr int kScoreThreads = 512;

__global__ void __launch_bounds__(kPoolMaxThreads)
pool_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
            float* __restrict__ q_mean, float* __restrict__ k_mean) {
  const int per_b = P.n_qblk + P.n_kblk;
  const int b = blockIdx.x / per_b;
  const int j = blockIdx.x % per_b;
  const bool is_q = j < P.n_qblk;
  const uint16_t* src = is_q ? q : k;
  const int blk = is_q ? P.block_q : P.block_k;
  const int n = is_q ? j : j - P.n_qblk;
  const int N = is_q ? P.n_qblk : P.n_kblk;
  float* dst = is_q ? q_mean : k_mean;
  const int l0 = n * blk;
  const int l1 = min(P.L, l0 + blk);
  const int HD = P.H * P.d;
  const float inv = 1.0f / static_cast<float>(l1 - l0);

  for (int vec = threadIdx.x; vec < HD / 8; vec += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const uint4* p = reinterpret_cast<const uint4*>(src + (static_cast<size_t>(b) * P.L + l0) * HD) + vec;
    const size_t stride = HD / 8;
    int l = l0;
    for (; l + 4 <= l1; l += 4) {
      uint4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = __ldg(p + (l - l0 + u) * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[0] += bf16_lo(x[u].x); acc[1] += bf16_hi(x[u].x);
        acc[2] += bf16_lo(x[u].y); acc[3] += bf16_hi(x[u].y);
        acc[4] += bf16_lo(x[u].z); acc[5] += bf16_hi(x[u].z);
        acc[6] += bf16_lo(x[u].w); acc[7] += bf16_hi(x[u].w);
      }
    }
    for (; l < l1; ++l) {
      uint4 x = __ldg(p + (l - l0) * stride);
      acc[0] += bf16_lo(x.x); acc[1] += bf16_hi(x.x);
      acc[2] += bf16_lo(x.y); acc[3] += bf16_hi(x.y);
      acc[4] += bf16_lo(x.z); acc[5] += bf16_hi(x.z);
      acc[6] += bf16_lo(x.w); acc[7] += bf16_hi(x.w);
    }
    const int h = (vec * 8) / P.d;
    const int c0 = (vec * 8) % P.d;
    float4* o = reinterpret_cast<float4*>(dst + ((static_cast<size_t>(b) * P.H + h) * N + n) * P.d + c0);
    o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

// Larger float <=> larger key; -0 is folded onto +0 first so equal scores tie.
__device__ __forceinline__ uint32_t order_key(float s) {
  if (s == 0.0f) s = 0.0f;
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kScoreThreads, 1)
score_select_kernel(Problem P, const float* __restrict__ q_mean, const float* __restrict__ k_mean,
                    int32_t* __restrict__ block_idx) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int D = P.d;
  const int NK = P.n_kblk;
  const int kt_stride = kKeyChunk + 1;
  float* sc = reinterpret_cast<float*>(smem);                 // [kRows][NK]
  float* qm = sc + kRows * NK;                                 // [kRows][D]
  float* kt = qm + kRows * D;                                  // [D][kKeyChunk + 1]  (phase 1)
  uint32_t* hist = reinterpret_cast<uint32_t*>(kt);            // [16 warps][256]     (phase 2)

  const int a0 = blockIdx.x * kRows;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * P.H + h;
  const int tid = threadIdx.x;

  for (int e = tid; e < kRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    qm[e] = (a0 + r < P.n_qblk) ? q_mean[(bh * P.n_qblk + a0 + r) * D + c] : 0.f;
  }

  // ---- phase 1: scores ----
  const int col = tid % kKeyChunk;
  const int rg = tid / kKeyChunk;          // rows 4*rg .. 4*rg+3
  for (int c0 = 0; c0 < NK; c0 += kKeyChunk) {
    __syncthreads();
    for (int e = tid; e < kKeyChunk * D; e += blockDim.x) {
      const int key = e / D, ch = e % D;
      kt[ch * kt_stride + key] = (c0 + key < NK) ? k_mean[(bh * NK + c0 + key) * D + ch] : 0.f;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* q0 = qm + (4 * rg) * D;
    for (int ch = 0; ch < D; ch += 4) {
      float kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) kv[u] = kt[(ch + u) * kt_stride + col];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 qv = *reinterpret_cast<const float4*>(q0 + i * D + ch);
        acc[i] = fmaf(qv.x, kv[0], acc[i]);
        acc[i] = fmaf(qv.y, kv[1], acc[i]);
        acc[i] = fmaf(qv.z, kv[2], acc[i]);
        acc[i] = fmaf(qv.w, kv[3], acc[i]);
      }
    }
    if (c0 + col < NK) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[(4 * rg + i) * NK + c0 + col] = acc[i];
    }
  }
  __syncthreads();

  // ---- phase 2: per-row radix select + ascending compaction ----
  const int warp = tid / 32;
  const int lane = tid % 32;
  const int a = a0 + warp;
  if (a >= P.n_qblk) return;
  const float* row = sc + warp * NK;
  uint32_t* hw = hist + warp * 256;
  const int keep = P.keep;

  uint32_t prefix = 0, pmask = 0;
  int remaining = keep;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int e = 0; e < 8; ++e) hw[lane * 8 + e] = 0;
    __syncwarp();
    for (int c = lane; c < NK; c += 32) {
      const uint32_t u = order_key(row[c]);
      if ((u & pmask) == prefix) atomicAdd(&hw[(u >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t bins[8];
    int mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bins[e] = hw[lane * 8 + e];
      mine += static_cast<int>(bins[e]);
    }
    int incl = mine;  // inclusive suffix sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const int above = incl - mine;
    const bool here = (above < remaining) && (incl >= remaining);
    const unsigned who = __ballot_sync(0xffffffffu, here);
    const int src = __ffs(who) - 1;
    int digit = 0, new_rem = 0;
    if (lane == src) {
      int cum = above;
      for (int e = 7; e >= 0; --e) {
        if (cum + static_cast<int>(bins[e]) >= remaining) {
          digit = lane * 8 + e;
          new_rem = remaining - cum;
          break;
        }
        cum += static_cast<int>(bins[e]);
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    remaining = __shfl_sync(0xffffffffu, new_rem, src);
    prefix |= static_cast<uint32_t>(digit) << shift;
    pmask |= 0xffu << shift;
    __syncwarp();
  }
  // prefix = key of the k-th best score; `remaining` of its ties are taken.
  int32_t* out = block_idx + (bh * P.n_qblk + a) * keep;
  int taken = 0, ties = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < NK; base += 32) {
    const int c = base + lane;
    const uint32_t u = c < NK ? order_key(row[c]) : 0u;
    const bool gt = c < NK && u > prefix;
    const bool eq = c < NK && u == prefix;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && ties + __popc(eqb & lt) < remaining);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = taken + __popc(tb & lt);
    if (take && pos < keep) out[pos] = c;
    taken += __popc(tb);
    ties += __popc(eqb);
  }
}

}  // namespace

size_t score_select_smem_bytes(const Problem& P) {
  const size_t phase1 = static_cast<size_t>(P.d) * (kKeyChunk + 1) * 4;
  const size_t phase2 = static_cast<size_t>(kScoreThreads / 32) * 256 * 4;
  return static_cast<size_t>(kRows) * P.n_kblk * 4 + static_cast<size_t>(kRows) * P.d * 4 +
         (phase1 > phase2 ? phase1 : phase2);
}

cudaError_t launch_block_select(const Problem& P, const uint16_t* q, const uint16_t* k, float* q_mean,
                                float* k_mean, int32_t* block_idx, cudaStream_t stream) {
  const int threads = (P.H * P.d / 8) < kPoolMaxThreads ? (P.H * P.d / 8) : kPoolMaxThreads;
  pool_kernel<<<P.B * (P.n_qblk + P.n_kblk), threads, 0, stream>>>(P, q, k, q_mean, k_mean);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = score_select_smem_bytes(P);
  e = cudaFuncSetAttribute(score_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((P.n_qblk + kRows - 1) / kRows, P.H, P.B);
  score_select_kernel<<<grid, kScoreThreads, smem, stream>>>(P, q_mean, k_mean, block_idx);
  return cudaGetLastError();
}

}  // namespace sda
