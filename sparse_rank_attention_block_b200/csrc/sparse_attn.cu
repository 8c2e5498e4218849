// Block-sparse attention A_M with optional gate epilogue (SparkDiffusion
// summary, robotworld.top, section 2.1: dense softmax(Q K^T / sqrt(d)) V
// restricted to the key blocks kept for each query block, then
// O = O_s + g r O_lr).
//
// Warp-level tensor-core kernel (mma.sync m16n8k16 bf16, fp32 accumulate):
// one CTA per (batch, head, query block), 16 query rows per warp, the kept
// 64-key blocks streamed through a two-stage cp.async ring. Online softmax in
// fp32 with exp2 and the 1/sqrt(d) scale folded into log2(e)/sqrt(d); a row
// lives in one quad of lanes, so row max / sum are quad shuffle reductions.
// Keys past L in a partial last block are masked to -inf. With a causal
// window a query block of chunk c attends to keys below the chunk's end only
// (the same mask, at that end) and keeps the first k_c entries of its row.
//
// Epilogue: O_s = O / l in fp32. With the gate, r_i = RMS(O_s,i) is taken from
// that unrounded fp32 row and O_s + g r O_lr is written as bf16.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kBK = 64;  // keys per block

template <int D>
__device__ __forceinline__ void load_tile(uint16_t* s, const uint16_t* __restrict__ gsrc, const Problem& P, int b,
                                          int h, int l0, int rows, int nthreads) {
  constexpr int CH = D / 8;
  for (int e = threadIdx.x; e < rows * CH; e += nthreads) {
    const int row = e / CH, ch = e % CH;
    const int l = l0 + row;
    const bool ok = l < P.L;
    const uint16_t* src = ok ? gsrc + ((static_cast<size_t>(b) * P.L + l) * P.H + h) * D + ch * 8 : gsrc;
    cp_async16(smem_u32(s + row * (D + 8) + ch * 8), src, ok ? 16 : 0);
  }
}

template <int D, int BQ>
__global__ void __launch_bounds__(BQ * 2)
sparse_attn_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                   const uint16_t* __restrict__ v, const int32_t* __restrict__ block_idx,
                   const uint16_t* __restrict__ o_lr, const float* __restrict__ gate, uint16_t* __restrict__ o,
                   unsigned* status) {
  constexpr int NTH = BQ * 2;
  constexpr int ST = D + 8;  // padded smem row (elements)
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);   // [BQ][ST]
  uint16_t* sK = sQ + BQ * ST;                          // [2][64][ST]
  uint16_t* sV = sK + 2 * kBK * ST;                     // [2][64][ST]

  const int a = blockIdx.x % P.n_qblk;
  const int h = (blockIdx.x / P.n_qblk) % P.H;
  const int b = blockIdx.x / (P.n_qblk * P.H);
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int g = lane / 4, t = lane % 4;
  const int q0 = qblk_start(P, a);
  const int q_end = qblk_end(P, a);          // rows of this block: [q0, q_end)
  const int cq = qblk_chunk(P, a);
  const int hi = chunk_end(P, cq);           // keys below hi are visible (L without a window)
  const int n_cand = chunk_cands(P, cq);
  const int keep = keep_of(P, n_cand);
  const int32_t* idx = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * P.keep;
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));

  auto block_of = [&](int j) -> int {
    const int kb = __ldg(idx + j);
    return (kb >= 0 && kb < n_cand) ? kb : -1;  // a candidate holds at least one visible key
  };

  load_tile<D>(sQ, q, P, b, h, q0, BQ, NTH);
  int kb_next = block_of(0);
  if (kb_next >= 0) {
    load_tile<D>(sK, k, P, b, h, kb_next * kBK, kBK, NTH);
    load_tile<D>(sV, v, P, b, h, kb_next * kBK, kBK, NTH);
  }
  cp_async_commit();

  uint32_t qf[D / 16][4];
  float acc[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool bad = false;

  for (int j = 0; j < keep; ++j) {
    const int st = j & 1;
    const int kb = kb_next;
    if (j + 1 < keep) {
      kb_next = block_of(j + 1);
      if (kb_next >= 0) {
        load_tile<D>(sK + (st ^ 1) * kBK * ST, k, P, b, h, kb_next * kBK, kBK, NTH);
        load_tile<D>(sV + (st ^ 1) * kBK * ST, v, P, b, h, kb_next * kBK, kBK, NTH);
      }
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        ldmatrix_x4(smem_u32(sQ + (16 * warp + (lane % 16)) * ST + 16 * ks + 8 * (lane / 16)), qf[ks][0], qf[ks][1],
                    qf[ks][2], qf[ks][3]);
    }
    if (kb < 0) {
      bad = true;
    } else {
      const uint16_t* cK = sK + st * kBK * ST;
      const uint16_t* cV = sV + st * kBK * ST;
      float s[kBK / 8][4];
#pragma unroll
      for (int nt = 0; nt < kBK / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < kBK / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(smem_u32(cK + (16 * np + (lane % 8) + 8 * (lane / 16)) * ST + 16 * ks + 8 * ((lane / 8) % 2)),
                      b0, b1, b2, b3);
          mma_bf16_16816(s[2 * np], qf[ks], b0, b1);
          mma_bf16_16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      const int valid = hi - kb * kBK;  // keys of this block that exist and are visible
      if (valid < kBK) {
#pragma unroll
        for (int nt = 0; nt < kBK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (8 * nt + 2 * t + (e & 1) >= valid) s[nt][e] = -INFINITY;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < kBK / 8; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0 * scale_log2);
      const float mn1 = fmaxf(m1, mx1 * scale_log2);
      const float al0 = exp2f(m0 - mn0);
      const float al1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < kBK / 8; ++nt) {
        s[nt][0] = exp2f(fmaf(s[nt][0], scale_log2, -mn0));
        s[nt][1] = exp2f(fmaf(s[nt][1], scale_log2, -mn0));
        s[nt][2] = exp2f(fmaf(s[nt][2], scale_log2, -mn1));
        s[nt][3] = exp2f(fmaf(s[nt][3], scale_log2, -mn1));
        rs0 += s[nt][0] + s[nt][1];
        rs1 += s[nt][2] + s[nt][3];
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        acc[nt][0] *= al0;
        acc[nt][1] *= al0;
        acc[nt][2] *= al1;
        acc[nt][3] *= al1;
      }
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(
              smem_u32(cV + (16 * kk + (lane % 8) + 8 * ((lane / 8) % 2)) * ST + 16 * np + 8 * (lane / 16)), b0, b1,
              b2, b3);
          mma_bf16_16816(acc[2 * np], pa, b0, b1);
          mma_bf16_16816(acc[2 * np + 1], pa, b2, b3);
        }
      }
    }
    __syncthreads();
  }
  if (bad && threadIdx.x == 0) report_status(status, kStatusBadIndex);

  // ---- epilogue ----
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    acc[nt][0] *= inv0;
    acc[nt][1] *= inv0;
    acc[nt][2] *= inv1;
    acc[nt][3] *= inv1;
  }
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  const int tok0 = q0 + r0, tok1 = q0 + r1;
  if (o_lr != nullptr) {
    float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      ss0 += acc[nt][0] * acc[nt][0] + acc[nt][1] * acc[nt][1];
      ss1 += acc[nt][2] * acc[nt][2] + acc[nt][3] * acc[nt][3];
    }
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
    const bool ok0 = tok0 < q_end, ok1 = tok1 < q_end;
    const size_t row0 = (static_cast<size_t>(b) * P.L + (ok0 ? tok0 : 0)) * P.H + h;
    const size_t row1 = (static_cast<size_t>(b) * P.L + (ok1 ? tok1 : 0)) * P.H + h;
    const float g0 = ok0 ? __ldg(gate + (P.gate_per_head ? row0 : row0 / P.H)) : 0.f;
    const float g1 = ok1 ? __ldg(gate + (P.gate_per_head ? row1 : row1 / P.H)) : 0.f;
    const float gr0 = g0 * sqrtf(ss0 / D), gr1 = g1 * sqrtf(ss1 / D);
    const uint32_t* lr0 = reinterpret_cast<const uint32_t*>(o_lr + row0 * D);
    const uint32_t* lr1 = reinterpret_cast<const uint32_t*>(o_lr + row1 * D);
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const uint32_t x0 = ok0 ? __ldg(lr0 + 4 * nt + t) : 0u;
      const uint32_t x1 = ok1 ? __ldg(lr1 + 4 * nt + t) : 0u;
      acc[nt][0] = fmaf(gr0, bf16_lo(x0), acc[nt][0]);
      acc[nt][1] = fmaf(gr0, bf16_hi(x0), acc[nt][1]);
      acc[nt][2] = fmaf(gr1, bf16_lo(x1), acc[nt][2]);
      acc[nt][3] = fmaf(gr1, bf16_hi(x1), acc[nt][3]);
    }
  }
  // stage the warp's 16 rows in sQ (its own rows, no longer needed) and store
  __syncwarp();
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    *reinterpret_cast<uint32_t*>(sQ + r0 * ST + 8 * nt + 2 * t) = pack_bf16(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<uint32_t*>(sQ + r1 * ST + 8 * nt + 2 * t) = pack_bf16(acc[nt][2], acc[nt][3]);
  }
  __syncwarp();
  constexpr int CH = D / 8;
  for (int e = lane; e < 16 * CH; e += 32) {
    const int row = 16 * warp + e / CH, ch = e % CH;
    const int l = q0 + row;
    if (l < q_end)
      *reinterpret_cast<uint4*>(o + ((static_cast<size_t>(b) * P.L + l) * P.H + h) * D + ch * 8) =
          *reinterpret_cast<const uint4*>(sQ + row * ST + ch * 8);
  }
}

template <int D, int BQ>
cudaError_t run(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* idx,
                const uint16_t* o_lr, const float* g, uint16_t* o, unsigned* status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(BQ + 4 * kBK) * (D + 8) * 2;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D, BQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>(P.B) * P.H * P.n_qblk;
  sparse_attn_kernel<D, BQ><<<blocks, BQ * 2, smem, stream>>>(P, q, k, v, idx, o_lr, g, o, status);
  return cudaGetLastError();
}

}  // namespace

size_t sparse_attn_smem_bytes(const Problem& P) {
  return static_cast<size_t>(P.block_q + 4 * kBK) * (P.d + 8) * 2;
}

cudaError_t launch_sparse_attn(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const int32_t* block_idx, const uint16_t* o_lr, const float* g, uint16_t* o,
                               unsigned* status, cudaStream_t stream) {
  // Plain O_s with 128-row query blocks runs on the tcgen05 kernel; 64-row
  // blocks (and the gate epilogue on a given O_lr) use the warp-MMA kernel below.
  if (o_lr == nullptr && sparse_attn_tc_supported(P))
    return launch_sparse_attn_tc(P, q, k, v, block_idx, o, status, stream);
  if (P.d == 128 && P.block_q == 128) return run<128, 128>(P, q, k, v, block_idx, o_lr, g, o, status, stream);
  if (P.d == 128 && P.block_q == 64) return run<128, 64>(P, q, k, v, block_idx, o_lr, g, o, status, stream);
  if (P.d == 64 && P.block_q == 128) return run<64, 128>(P, q, k, v, block_idx, o_lr, g, o, status, stream);
  if (P.d == 64 && P.block_q == 64) return run<64, 64>(P, q, k, v, block_idx, o_lr, g, o, status, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sda
