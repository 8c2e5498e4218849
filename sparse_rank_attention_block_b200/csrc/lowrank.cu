// Low-rank branch of the compensated sparse attention (SparkDiffusion summary,
// robotworld.top, section 2.1: features, global state, readout):
//
//   k~_j = R_r(p_j) phi(P_k k_j),  C = sum_j k~_j v_j^T          (state kernels)
//   q~_i = R_r(p_i) phi(P_q q_i),  O_lr,i = RMSNorm(q~_i^T C)   (readout kernel)
//
// Both passes stream [B, L, H, d] bf16 tensors once and are HBM-bound; the
// per-token products (P x: 2rd flop, k~ v^T / q~^T C: 2rd flop each) run on
// the tensor cores (mma.sync m16n8k16 bf16, fp32 accumulate) so that the
// arithmetic hides under the memory stream. Features are kept to ~16 bits by
// splitting them (and C) into a bf16 head and a bf16 tail and issuing one MMA
// per significant product, which keeps the branch within fp32-level error.
//
// State: one CTA per (batch, head, token piece) accumulates a partial r x d
// state in registers; a second kernel sums the pieces in a fixed order
// (deterministic, no float atomics) and also emits C^T split into bf16
// head/tail, the operand layout the readout MMAs consume. With a causal
// window the pieces follow the chunks and the sum is a prefix sum: the state
// of chunk c covers the pieces of chunks 0..c, and a chunk-c query reads it.
//
// Rotation angles come from a table of cos/sin per (axis coordinate, pair)
// built once per call in double precision (rope_table_kernel).

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kTile = 64;          // tokens per sub-tile (4 warps x 16)
constexpr int kThreads = 128;
constexpr int kReadoutTiles = 4;   // sub-tiles per readout CTA

__global__ void rope_table_kernel(Problem P, float2* tab) { build_rope_table(P, tab); }

template <int D>
__device__ __forceinline__ void load_rows(uint16_t* s, const uint16_t* __restrict__ g, const Problem& P, int b,
                                          int h, int l0, int l_end) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int e = threadIdx.x; e < kTile * CH; e += blockDim.x) {
    const int row = e / CH, ch = e % CH;
    const int l = l0 + row;
    const bool ok = l < l_end;
    const uint16_t* src = ok ? g + ((static_cast<size_t>(b) * P.L + l) * P.H + h) * D + ch * 8 : g;
    cp_async16(smem_u32(s + row * (D + 8) + ch * 8), src, ok ? 16 : 0);
  }
}

template <int D, int R>
__device__ __forceinline__ void load_proj(uint16_t* s, const uint16_t* __restrict__ p) {
  constexpr int CH = D / 8;
  for (int e = threadIdx.x; e < R * CH; e += blockDim.x) {
    const int row = e / CH, ch = e % CH;
    cp_async16(smem_u32(s + row * (D + 8) + ch * 8), p + row * D + ch * 8, 16);
  }
}

// U = X_rows(16) . P^T for the warp's 16 rows of the tile in `sx`, then
// phi and RoPE: returns the features in mma accumulator layout (fp32).
template <int D, int R>
__device__ __forceinline__ void features_16(const uint16_t* sx, const uint16_t* sp, const Problem& P,
                                            const float2* __restrict__ tab, int l_row0, int l_end,
                                            float (&u)[R / 8][4]) {
  const int lane = threadIdx.x % 32;
  const int warp = threadIdx.x / 32;
#pragma unroll
  for (int nt = 0; nt < R / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) u[nt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    ldmatrix_x4(smem_u32(sx + (16 * warp + (lane % 16)) * (D + 8) + 16 * ks + 8 * (lane / 16)), a[0], a[1], a[2],
                a[3]);
#pragma unroll
    for (int np = 0; np < R / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(smem_u32(sp + (16 * np + (lane % 8) + 8 * (lane / 16)) * (D + 8) + 16 * ks + 8 * ((lane / 8) % 2)),
                  b0, b1, b2, b3);
      mma_bf16_16816(u[2 * np], a, b0, b1);
      mma_bf16_16816(u[2 * np + 1], a, b2, b3);
    }
  }
  const int g = lane / 4, t = lane % 4;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int l = l_row0 + 16 * warp + g + 8 * half;
    const bool ok = l < l_end;
#pragma unroll
    for (int nt = 0; nt < R / 8; ++nt) {
      const int m = 4 * nt + t;  // rotation pair of columns (8nt + 2t, 8nt + 2t + 1)
      const float x = elu_plus_one(u[nt][2 * half]);
      const float y = elu_plus_one(u[nt][2 * half + 1]);
      const float2 cs = ok ? rope_lookup(P, tab, l, m) : make_float2(0.f, 0.f);
      u[nt][2 * half] = x * cs.x - y * cs.y;
      u[nt][2 * half + 1] = x * cs.y + y * cs.x;
    }
  }
}

// ---------------------------------------------------------------------------
// state: partial C over one token chunk
// ---------------------------------------------------------------------------

template <int D, int R>
__global__ void __launch_bounds__(kThreads)
lowrank_state_kernel(Problem P, int split_len, int n_split, int n_sub, const float2* __restrict__ tab,
                     const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                     const uint16_t* __restrict__ p_k, float* __restrict__ c_part) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sP = reinterpret_cast<uint16_t*>(smem);                 // [R][D+8]
  uint16_t* sK = sP + R * (D + 8);                                  // [2][64][D+8]
  uint16_t* sV = sK + 2 * kTile * (D + 8);                          // [2][64][D+8]
  uint16_t* sHi = sV + 2 * kTile * (D + 8);                         // [64][R+8]
  uint16_t* sLo = sHi + kTile * (R + 8);                            // [64][R+8]

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int c = s / n_sub;  // causal chunk of this piece (0 without a window)
  const int l_begin = c * P.chunk_tokens + (s - c * n_sub) * split_len;
  const int l_end = min(chunk_end(P, c), l_begin + split_len);  // may be empty: the partial state is zero
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int g = lane / 4, t = lane % 4;
  constexpr int NT = D / 32;          // n-tiles of 8 channels per warp
  const int n0 = warp * (D / 4);

  float acc[R / 16][NT][4];
#pragma unroll
  for (int mt = 0; mt < R / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

  const int tiles = l_end > l_begin ? (l_end - l_begin + kTile - 1) / kTile : 0;
  load_proj<D, R>(sP, p_k);
  if (tiles > 0) {
    load_rows<D>(sK, k, P, b, h, l_begin, l_end);
    load_rows<D>(sV, v, P, b, h, l_begin, l_end);
  }
  cp_async_commit();

  for (int it = 0; it < tiles; ++it) {
    const int st = it & 1;
    if (it + 1 < tiles) {
      const int l0n = l_begin + (it + 1) * kTile;
      load_rows<D>(sK + (st ^ 1) * kTile * (D + 8), k, P, b, h, l0n, l_end);
      load_rows<D>(sV + (st ^ 1) * kTile * (D + 8), v, P, b, h, l0n, l_end);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint16_t* cK = sK + st * kTile * (D + 8);
    const uint16_t* cV = sV + st * kTile * (D + 8);
    const int l0 = l_begin + it * kTile;

    float u[R / 8][4];
    features_16<D, R>(cK, sP, P, tab, l0, l_end, u);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = 16 * warp + g + 8 * half;
#pragma unroll
      for (int nt = 0; nt < R / 8; ++nt) {
        float h0, t0, h1, t1;
        split_bf16(u[nt][2 * half], h0, t0);
        split_bf16(u[nt][2 * half + 1], h1, t1);
        *reinterpret_cast<uint32_t*>(sHi + row * (R + 8) + 8 * nt + 2 * t) = pack_bf16(h0, h1);
        *reinterpret_cast<uint32_t*>(sLo + row * (R + 8) + 8 * nt + 2 * t) = pack_bf16(t0, t1);
      }
    }
    __syncthreads();

    // C[r x d] += k~^T (r x 64) . V (64 x d); this warp owns channels [n0, n0 + D/4).
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk) {
      uint32_t ahi[R / 16][4], alo[R / 16][4];
#pragma unroll
      for (int mt = 0; mt < R / 16; ++mt) {
        const int off = (16 * kk + (lane % 8) + 8 * (lane / 16)) * (R + 8) + 16 * mt + 8 * ((lane / 8) % 2);
        ldmatrix_x4_trans(smem_u32(sHi + off), ahi[mt][0], ahi[mt][1], ahi[mt][2], ahi[mt][3]);
        ldmatrix_x4_trans(smem_u32(sLo + off), alo[mt][0], alo[mt][1], alo[mt][2], alo[mt][3]);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(
            smem_u32(cV + (16 * kk + (lane % 8) + 8 * ((lane / 8) % 2)) * (D + 8) + n0 + 16 * np + 8 * (lane / 16)),
            b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < R / 16; ++mt) {
          mma_bf16_16816(acc[mt][2 * np], ahi[mt], b0, b1);
          mma_bf16_16816(acc[mt][2 * np], alo[mt], b0, b1);
          mma_bf16_16816(acc[mt][2 * np + 1], ahi[mt], b2, b3);
          mma_bf16_16816(acc[mt][2 * np + 1], alo[mt], b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();  // an empty piece still issued the projection load

  float* out = c_part + ((static_cast<size_t>(b) * P.H + h) * n_split + s) * R * D;
#pragma unroll
  for (int mt = 0; mt < R / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int col = n0 + 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(out + (16 * mt + g) * D + col) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
      *reinterpret_cast<float2*>(out + (16 * mt + g + 8) * D + col) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
    }
}

// Sum the partials in piece order; after the n_sub pieces of each chunk write
// that chunk's (prefix) state: C (fp32 [r][d]), C^T in fp32 ([d][r]) and C^T
// as a bf16 head/tail pair ([d][r] each) for the readout MMAs. Without a
// window there is one chunk and this is the plain sum over all pieces.
__global__ void lowrank_reduce_kernel(Problem P, int n_split, int n_sub, const float* __restrict__ c_part,
                                      float* __restrict__ c_state, float* __restrict__ c_out,
                                      float* __restrict__ ct_f32, uint16_t* __restrict__ ct_hi,
                                      uint16_t* __restrict__ ct_lo) {
  const int bh = blockIdx.y;
  const int RD = P.rank * P.d;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // one element of C per thread
  if (e < RD) {
    const float* src = c_part + static_cast<size_t>(bh) * n_split * RD + e;
    const int m = e / P.d, n = e % P.d;
    // fixed summation order (piece 0, 1, ...); loads issued 8 at a time
    float s = 0.f;
    int i = 0;
    for (int c = 0; c < P.n_chunks; ++c) {
      const int i_end = (c + 1) * n_sub;
      for (; i + 8 <= i_end; i += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = __ldg(src + static_cast<size_t>(i + u) * RD);
#pragma unroll
        for (int u = 0; u < 8; ++u) s += x[u];
      }
      for (; i < i_end; ++i) s += __ldg(src + static_cast<size_t>(i) * RD);
      const size_t o = (static_cast<size_t>(bh) * P.n_chunks + c) * RD;
      c_state[o + e] = s;
      if (c_out) c_out[o + e] = s;
      if (ct_f32) ct_f32[o + n * P.rank + m] = s;
      float hd, tl;
      split_bf16(s, hd, tl);
      __nv_bfloat16 hb = __float2bfloat16_rn(hd), tb = __float2bfloat16_rn(tl);
      ct_hi[o + n * P.rank + m] = *reinterpret_cast<uint16_t*>(&hb);
      ct_lo[o + n * P.rank + m] = *reinterpret_cast<uint16_t*>(&tb);
    }
  }
}

// ---------------------------------------------------------------------------
// readout: O_lr = RMSNorm(q~^T C)
// ---------------------------------------------------------------------------

template <int D, int R>
__global__ void __launch_bounds__(kThreads)
lowrank_readout_kernel(Problem P, const float2* __restrict__ tab, const uint16_t* __restrict__ q,
                       const uint16_t* __restrict__ p_q, const uint16_t* __restrict__ ct_hi,
                       const uint16_t* __restrict__ ct_lo, uint16_t* __restrict__ o_lr) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sP = reinterpret_cast<uint16_t*>(smem);                 // [R][D+8]
  uint16_t* sQ = sP + R * (D + 8);                                  // [2][64][D+8]
  uint16_t* sCh = sQ + 2 * kTile * (D + 8);                         // [D][R+8]
  uint16_t* sCl = sCh + D * (R + 8);                                // [D][R+8]

  const int h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int g = lane / 4, t = lane % 4;
  // blockIdx.x = (causal chunk, run of kReadoutTiles tiles inside it); rows of
  // chunk c read its state C_c (one chunk, the whole sequence, without a window)
  const int per_chunk = (P.chunk_tokens + kReadoutTiles * kTile - 1) / (kReadoutTiles * kTile);
  const int c = blockIdx.x / per_chunk;
  const size_t bh = (static_cast<size_t>(b) * P.H + h) * P.n_chunks + c;
  const int l_first = c * P.chunk_tokens + (blockIdx.x - c * per_chunk) * kReadoutTiles * kTile;
  const int l_last = min(chunk_end(P, c), l_first + kReadoutTiles * kTile);
  if (l_first >= l_last) return;  // uniform over the CTA
  const int tiles = (l_last - l_first + kTile - 1) / kTile;

  load_proj<D, R>(sP, p_q);
  {
    constexpr int CH = R / 8;
    for (int e = threadIdx.x; e < D * CH; e += blockDim.x) {
      const int row = e / CH, ch = e % CH;
      cp_async16(smem_u32(sCh + row * (R + 8) + ch * 8), ct_hi + bh * R * D + row * R + ch * 8, 16);
      cp_async16(smem_u32(sCl + row * (R + 8) + ch * 8), ct_lo + bh * R * D + row * R + ch * 8, 16);
    }
  }
  load_rows<D>(sQ, q, P, b, h, l_first, l_last);
  cp_async_commit();

  for (int it = 0; it < tiles; ++it) {
    const int st = it & 1;
    uint16_t* cQ = sQ + st * kTile * (D + 8);
    if (it + 1 < tiles) {
      load_rows<D>(sQ + (st ^ 1) * kTile * (D + 8), q, P, b, h, l_first + (it + 1) * kTile, l_last);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int l0 = l_first + it * kTile;

    float u[R / 8][4];
    features_16<D, R>(cQ, sP, P, tab, l0, l_last, u);
    uint32_t ahi[R / 16][4], alo[R / 16][4];
#pragma unroll
    for (int ks = 0; ks < R / 16; ++ks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* src = u[2 * ks + (e >> 1)] + 2 * (e & 1);
        float h0, t0, h1, t1;
        split_bf16(src[0], h0, t0);
        split_bf16(src[1], h1, t1);
        ahi[ks][e] = pack_bf16(h0, h1);
        alo[ks][e] = pack_bf16(t0, t1);
      }
    }
    float x[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < R / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int off = (16 * np + (lane % 8) + 8 * (lane / 16)) * (R + 8) + 16 * ks + 8 * ((lane / 8) % 2);
        uint32_t h0, h1, h2, h3, c0, c1, c2, c3;
        ldmatrix_x4(smem_u32(sCh + off), h0, h1, h2, h3);
        ldmatrix_x4(smem_u32(sCl + off), c0, c1, c2, c3);
        mma_bf16_16816(x[2 * np], ahi[ks], h0, h1);
        mma_bf16_16816(x[2 * np], alo[ks], h0, h1);
        mma_bf16_16816(x[2 * np], ahi[ks], c0, c1);
        mma_bf16_16816(x[2 * np + 1], ahi[ks], h2, h3);
        mma_bf16_16816(x[2 * np + 1], alo[ks], h2, h3);
        mma_bf16_16816(x[2 * np + 1], ahi[ks], c2, c3);
      }
    }
    // RMSNorm over the d channels of rows g and g+8 (a row lives in one quad).
    float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      ss0 += x[nt][0] * x[nt][0] + x[nt][1] * x[nt][1];
      ss1 += x[nt][2] * x[nt][2] + x[nt][3] * x[nt][3];
    }
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
    const float inv0 = rsqrtf(ss0 / D + P.rms_eps);
    const float inv1 = rsqrtf(ss1 / D + P.rms_eps);
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      *reinterpret_cast<uint32_t*>(cQ + (16 * warp + g) * (D + 8) + 8 * nt + 2 * t) =
          pack_bf16(x[nt][0] * inv0, x[nt][1] * inv0);
      *reinterpret_cast<uint32_t*>(cQ + (16 * warp + g + 8) * (D + 8) + 8 * nt + 2 * t) =
          pack_bf16(x[nt][2] * inv1, x[nt][3] * inv1);
    }
    __syncwarp();
    constexpr int CH = D / 8;
    for (int e = lane; e < 16 * CH; e += 32) {
      const int row = 16 * warp + e / CH, ch = e % CH;
      const int l = l0 + row;
      if (l < l_last) {
        const uint4 val = *reinterpret_cast<const uint4*>(cQ + row * (D + 8) + ch * 8);
        *reinterpret_cast<uint4*>(o_lr + ((static_cast<size_t>(b) * P.L + l) * P.H + h) * D + ch * 8) = val;
      }
    }
    __syncthreads();
  }
}

template <int D, int R>
size_t state_smem() {
  return (static_cast<size_t>(R) * (D + 8) + 4 * kTile * (D + 8) + 2 * kTile * (R + 8)) * 2;
}
template <int D, int R>
size_t readout_smem() {
  return (static_cast<size_t>(R) * (D + 8) + 2 * kTile * (D + 8) + 2 * D * (R + 8)) * 2;
}

template <int D, int R>
cudaError_t run_state(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                      const uint16_t* v, const uint16_t* p_k, float* c_part, float* c_state, float* c_out,
                      float* ct_f32, uint16_t* ct_hi, uint16_t* ct_lo, unsigned* status, bool use_tc,
                      uint16_t* k_mean, cudaStream_t stream) {
  cudaError_t e;
  if (use_tc && lowrank_state_tc_supported(P)) {
    e = launch_lowrank_state_tc(P, lay, tab, k, k_mean, v, p_k, c_part, status, stream);
  } else {
    const size_t smem = state_smem<D, R>();
    e = cudaFuncSetAttribute(lowrank_state_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(lay.n_split, P.H, P.B);
    lowrank_state_kernel<D, R><<<grid, kThreads, smem, stream>>>(P, lay.split_len, lay.n_split, lay.n_sub, tab, k,
                                                                 v, p_k, c_part);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  lowrank_reduce_kernel<<<dim3((P.rank * P.d + 127) / 128, P.B * P.H), 128, 0, stream>>>(
      P, lay.n_split, lay.n_sub, c_part, c_state, c_out, ct_f32, ct_hi, ct_lo);
  return cudaGetLastError();
}

template <int D, int R>
cudaError_t run_readout(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                        const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr, cudaStream_t stream) {
  const size_t smem = readout_smem<D, R>();
  cudaError_t e = cudaFuncSetAttribute(lowrank_readout_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int per_chunk = (P.chunk_tokens + kReadoutTiles * kTile - 1) / (kReadoutTiles * kTile);
  dim3 grid(per_chunk * P.n_chunks, P.H, P.B);
  lowrank_readout_kernel<D, R><<<grid, kThreads, smem, stream>>>(P, tab, q, p_q, ct_hi, ct_lo, o_lr);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_table(const Problem& P, float2* tab, cudaStream_t stream) {
  rope_table_kernel<<<1, 256, 0, stream>>>(P, tab);
  return cudaGetLastError();
}

#define SDA_DISPATCH_DR(D_, R_, CALL)                                      \
  do {                                                                     \
    if ((D_) == 64 && (R_) == 16) return CALL(64, 16);                      \
    if ((D_) == 64 && (R_) == 32) return CALL(64, 32);                      \
    if ((D_) == 64 && (R_) == 64) return CALL(64, 64);                      \
    if ((D_) == 128 && (R_) == 16) return CALL(128, 16);                    \
    if ((D_) == 128 && (R_) == 32) return CALL(128, 32);                    \
    if ((D_) == 128 && (R_) == 64) return CALL(128, 64);                    \
  } while (0)

cudaError_t launch_lowrank_state(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                                 const uint16_t* v, const uint16_t* p_k, float* c_part, float* c_state,
                                 float* c_out, float* ct_f32, uint16_t* ct_hi, uint16_t* ct_lo,
                                 unsigned* status, bool use_tc, uint16_t* k_mean, cudaStream_t stream) {
#define SDA_CALL_STATE(D, R) \
  run_state<D, R>(P, lay, tab, k, v, p_k, c_part, c_state, c_out, ct_f32, ct_hi, ct_lo, status, use_tc, k_mean, stream)
  SDA_DISPATCH_DR(P.d, P.rank, SDA_CALL_STATE);
#undef SDA_CALL_STATE
  return cudaErrorInvalidValue;
}

cudaError_t launch_lowrank_readout(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                                   const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr, unsigned* status,
                                   bool use_tc, cudaStream_t stream) {
  if (use_tc && lowrank_readout_tc_supported(P))
    return launch_lowrank_readout_tc(P, tab, q, p_q, ct_hi, ct_lo, o_lr, status, stream);
#define SDA_CALL_READOUT(D, R) run_readout<D, R>(P, tab, q, p_q, ct_hi, ct_lo, o_lr, stream)
  SDA_DISPATCH_DR(P.d, P.rank, SDA_CALL_READOUT);
#undef SDA_CALL_READOUT
  return cudaErrorInvalidValue;
}

size_t lowrank_state_smem_bytes(const Problem& P) {
  return (static_cast<size_t>(P.rank) * (P.d + 8) + 4 * kTile * (P.d + 8) + 2 * kTile * (P.rank + 8)) * 2;
}
size_t lowrank_readout_smem_bytes(const Problem& P) {
  return (static_cast<size_t>(P.rank) * (P.d + 8) + 2 * kTile * (P.d + 8) + 2 * P.d * (P.rank + 8)) * 2;
}

}  // namespace sda
