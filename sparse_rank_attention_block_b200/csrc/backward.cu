// Backward of the compensated sparse attention (training needs it: the sparse
// warm-up adds the low-rank projections and the gate as trained parameters and
// backpropagates through the sparse attention; H3 portability report, sections
// 2.1-2.2; forward equations: SparkDiffusion summary, robotworld.top, section 2.1).
//
// Given dO for O = O_s + g r O_lr (r = RMS(O_s), O_lr = RMSNorm(q~^T C)), the
// chain rule taken step by step in reverse:
//   gate      dO_s = dO + g (dO . O_lr) O_s / (d r),  dO_lr = g r dO,  dg = r (dO . O_lr)
//   readout   dX = (dO_lr - y mean(dO_lr y)) / rho  (y = O_lr),  dq~ = C dX,  dC = sum_i q~_i dX_i^T
//   features  dU = R^T dq~ * phi'(U),  dq += dU P_q,  dP_q = sum dU q^T   (same on the k side)
//   state     dv += dC^T k~,  dk~ = dC v
//   sparse    P = softmax(s), D_i = dO_s,i . O_s,i,  dS = P (dO_s V^T - D),
//             dq += dS K / sqrt(d),  dk += dS^T Q / sqrt(d),  dv += P^T dO_s
// with the forward's block map held fixed.
//
// The low-rank and gate parts are fp32 SIMT kernels, one warp per row with the
// channels split over the lanes; the forward quantities (C, O_s, O_lr) come
// from the forward kernels. The sparse branch runs on the tensor cores
// (backward_tc.cu) at d = 128 with 128-row query blocks -- the forward then
// also leaves each row's log-sum-exp and the gate kernel D = dO_s . O_s and a
// bf16 copy of dO_s -- and on the SIMT kernels below otherwise. Every sum has a fixed order (no float atomics):
// dK/dV walk a transposed map (the query blocks that kept each key block, in
// ascending order), dC, dP_q and dP_k are chunked outer-product sums reduced
// in chunk order. No kernel waits on another CTA.

#include "common.cuh"
#include "kernels.h"

namespace sda {

namespace {

constexpr int kRowWarps = 8;           // warps (rows in flight) per CTA of the row kernels
constexpr int kOuterRows = 1024;       // rows per partial of the outer-product sums
constexpr int kOuterThreads = 256;

__device__ __forceinline__ float bf(const uint16_t* p) { return __uint_as_float(static_cast<uint32_t>(*p) << 16); }
__device__ __forceinline__ float elu1(float u) { return u > 0.f ? u + 1.f : expf(u); }
__device__ __forceinline__ float elu1_prime(float u) { return u > 0.f ? 1.f : expf(u); }

// ---------------------------------------------------------------------------
// gate: one warp per token, heads in order (dg summed over heads in that order)
// ---------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_gate_kernel(Problem P, const uint16_t* __restrict__ o_s, const uint16_t* __restrict__ o_lr,
                const float* __restrict__ g, const uint16_t* __restrict__ d_o, float* __restrict__ do_s,
                float* __restrict__ do_lr, float* __restrict__ dg, uint16_t* __restrict__ do_s_bf,
                float* __restrict__ dd) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x % 32;
  const long long tok = static_cast<long long>(blockIdx.x) * kRowWarps + threadIdx.x / 32;
  if (tok >= static_cast<long long>(P.B) * P.L) return;
  float dg_tok = 0.f;
  for (int h = 0; h < P.H; ++h) {
    const size_t row = static_cast<size_t>(tok) * P.H + h;
    float os[E], ol[E], dy[E];
    float ss = 0.f, dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const size_t c = row * D + lane + 32 * e;
      os[e] = bf(o_s + c);
      ol[e] = bf(o_lr + c);
      dy[e] = bf(d_o + c);
      ss += os[e] * os[e];
      dot += dy[e] * ol[e];
    }
    ss = warp_sum(ss);
    dot = warp_sum(dot);
    const float r = sqrtf(ss / D);
    const float gh = __ldg(g + (P.gate_per_head ? row : static_cast<size_t>(tok)));
    const float coef = r > 0.f ? gh * dot / (D * r) : 0.f;
    float dsum = 0.f;  // D = dO_s . O_s of the row (softmax backward)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const size_t c = row * D + lane + 32 * e;
      const float ds = dy[e] + coef * os[e];
      if (do_s != nullptr) do_s[c] = ds;  // fp32 copy for the SIMT sparse kernels
      do_lr[c] = gh * r * dy[e];
      dsum += ds * os[e];
      if (do_s_bf != nullptr) do_s_bf[c] = __bfloat16_as_ushort(__float2bfloat16_rn(ds));
    }
    dsum = warp_sum(dsum);
    if (dd != nullptr && lane == 0) dd[row] = dsum;
    if (P.gate_per_head) {
      if (lane == 0) dg[row] = r * dot;
    } else {
      dg_tok += r * dot;
    }
  }
  if (!P.gate_per_head && lane == 0) dg[tok] = dg_tok;
}

// ---------------------------------------------------------------------------
// low-rank features: a row's r-vectors live one element per lane (m = lane + 32 w)
// ---------------------------------------------------------------------------

// [R][D] fp32 matrices in shared memory are stored lane-major: element (m, c)
// at m * D + (c % 32) * (D / 32) + c / 32, so the D / 32 channels lane + 32 e
// a lane works on are one vector load.
template <int D>
__device__ __forceinline__ int lane_major(int i) {
  const int m = i / D, c = i % D;
  return m * D + (c % 32) * (D / 32) + c / 32;
}
template <int D>
__device__ __forceinline__ void ld_lane(const float* src, float (&out)[D / 32]) {
  if constexpr (D / 32 == 4) {
    const float4 v = *reinterpret_cast<const float4*>(src);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(src);
    out[0] = v.x; out[1] = v.y;
  }
}

// Token rows per warp of the low-rank kernels (every element of P, C or G a
// warp reads from shared memory serves all of them). One row measured fastest:
// four rows cut those reads fourfold but need 175-190 registers, which leaves
// one CTA per SM, and the reduce-scatter chains then stall (query side at the
// 720P layer 9.8 ms against 7.4 ms).
constexpr int kLrRows = 1;

// y[n]_m = sum_c A[m][c] x[n]_c for m < R and the warp's NR rows (A lane-major
// [R][D] in shared memory, x[n] the channels lane + 32 e of row n); y[n]_m
// lands in lane m % 32, element m / 32. Per group of 32 outputs a warp
// reduce-scatter: every lane forms partial sums over its channels, then five
// butterfly stages each halve the values a lane keeps (31 shuffles per row,
// additions in a fixed order). The first stage is taken as the pairs
// (m, m + 16) are formed, so at most 16 partials per row are live.
template <int D, int R, int NR>
__device__ __forceinline__ void matvec_rs(const float* sA, const float (&x)[NR][D / 32],
                                          float (&y)[NR][(R + 31) / 32], int lane) {
  constexpr int E = D / 32, W = (R + 31) / 32;
  auto row_of = [&](int m, float (&a)[E]) {
    if (m < R) {
      ld_lane<D>(sA + m * D + lane * E, a);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) a[e] = 0.f;
    }
  };
#pragma unroll
  for (int w = 0; w < W; ++w) {
    float v[NR][16];
    const bool hi16 = (lane & 16) != 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float alo[E], aup[E];
      row_of(32 * w + j, alo);
      row_of(32 * w + j + 16, aup);
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        float lo = 0.f, up = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          lo = fmaf(alo[e], x[n][e], lo);
          up = fmaf(aup[e], x[n][e], up);
        }
        v[n][j] = (hi16 ? up : lo) + __shfl_xor_sync(0xffffffffu, hi16 ? lo : up, 16);
      }
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      const bool hi = (lane & o) != 0;
#pragma unroll
      for (int n = 0; n < NR; ++n) {
#pragma unroll
        for (int j = 0; j < o; ++j) {
          const float keep = hi ? v[n][j + o] : v[n][j];
          const float send = hi ? v[n][j] : v[n][j + o];
          v[n][j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NR; ++n) y[n][w] = v[n][0];
  }
}

// out[n]_c += sum_m y[n]_m A[m][c] for the rows' channels (y[n] one element per lane).
template <int D, int R, int NR>
__device__ __forceinline__ void vecmat(const float* sA, const float (&y)[NR][(R + 31) / 32],
                                       float (&out)[NR][D / 32], int lane) {
  constexpr int E = D / 32, W = (R + 31) / 32;
#pragma unroll
  for (int w = 0; w < W; ++w) {
#pragma unroll 4
    for (int mm = 0; mm < (R < 32 ? R : 32); ++mm) {
      float a[E];
      ld_lane<D>(sA + (32 * w + mm) * D + lane * E, a);
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const float t = __shfl_sync(0xffffffffu, y[n][w], mm);
#pragma unroll
        for (int e = 0; e < E; ++e) out[n][e] = fmaf(t, a[e], out[n][e]);
      }
    }
  }
}

// cos / sin of element m's pair for token l (lanes with m >= R get the identity).
__device__ __forceinline__ float2 pair_rot(const Problem& P, const float2* tab, int l, int m) {
  return m < P.rank ? rope_lookup(P, tab, l, m >> 1) : make_float2(1.f, 0.f);
}

// x~ = R phi(u): element m pairs with m ^ 1, held by lane ^ 1.
template <int R>
__device__ __forceinline__ void features(const Problem& P, const float2* tab, int l, const float (&u)[(R + 31) / 32],
                                         float (&f)[(R + 31) / 32], int lane) {
  constexpr int W = (R + 31) / 32;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int m = lane + 32 * w;
    const float mine = elu1(u[w]);
    const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
    const float2 cs = pair_rot(P, tab, l, m);
    f[w] = (m & 1) ? other * cs.y + mine * cs.x : mine * cs.x - other * cs.y;
  }
}

// du = R^T dx~ * phi'(u): the transpose of a rotation by a turns by -a.
template <int R>
__device__ __forceinline__ void features_back(const Problem& P, const float2* tab, int l,
                                              const float (&u)[(R + 31) / 32], const float (&dxt)[(R + 31) / 32],
                                              float (&du)[(R + 31) / 32], int lane) {
  constexpr int W = (R + 31) / 32;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int m = lane + 32 * w;
    const float mine = dxt[w];
    const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
    const float2 cs = pair_rot(P, tab, l, m);
    const float rot = (m & 1) ? -other * cs.y + mine * cs.x : mine * cs.x + other * cs.y;
    du[w] = m < R ? rot * elu1_prime(u[w]) : 0.f;
  }
}

// Query side of the low-rank branch, kLrRows tokens of a (batch, head) per
// warp: recompute U, q~, X and rho; dX (in place of dO_lr), dq~, dU,
// dq = dU P_q. Writes q~ and dU rows for the dC and dP_q sums. A CTA takes
// tok_per_cta tokens of one causal chunk (of the sequence without a window),
// whose rows read that chunk's prefix state. Rows past the CTA's range are
// computed on its last token and not stored.
template <int D, int R>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_lr_q_kernel(Problem P, const float2* __restrict__ tab, const uint16_t* __restrict__ q,
                const uint16_t* __restrict__ p_q, const float* __restrict__ c_state, float* __restrict__ dx,
                float* __restrict__ dq, float* __restrict__ qt_rows, float* __restrict__ du_rows, int tok_per_cta) {
  constexpr int E = D / 32, W = (R + 31) / 32, NR = kLrRows;
  extern __shared__ float bwd_smem[];
  float* sP = bwd_smem;           // P_q, fp32 [R][D]
  float* sC = bwd_smem + R * D;   // C of this (batch, head, chunk), fp32 [R][D]
  const int h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int tiles = (P.chunk_tokens + tok_per_cta - 1) / tok_per_cta;
  const int c = blockIdx.x / tiles;
  const size_t bhc = (static_cast<size_t>(b) * P.H + h) * P.n_chunks + c;
  for (int i = threadIdx.x; i < R * D; i += blockDim.x) {
    sP[lane_major<D>(i)] = bf(p_q + i);
    sC[lane_major<D>(i)] = c_state[bhc * R * D + i];
  }
  __syncthreads();
  const int l0 = c * P.chunk_tokens + (blockIdx.x % tiles) * tok_per_cta;
  const int l1 = min(chunk_end(P, c), l0 + tok_per_cta);
  for (int lb = l0 + warp * NR; lb < l1; lb += kRowWarps * NR) {
    int ls[NR];
    size_t row[NR];
    float x[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      ls[n] = min(lb + n, l1 - 1);
      row[n] = (static_cast<size_t>(b) * P.L + ls[n]) * P.H + h;
#pragma unroll
      for (int e = 0; e < E; ++e) x[n][e] = bf(q + row[n] * D + lane + 32 * e);
    }
    float u[NR][W], qt[NR][W];
    matvec_rs<D, R, NR>(sP, x, u, lane);
#pragma unroll
    for (int n = 0; n < NR; ++n) features<R>(P, tab, ls[n], u[n], qt[n], lane);
    float X[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int e = 0; e < E; ++e) X[n][e] = 0.f;
    vecmat<D, R, NR>(sC, qt, X, lane);
    float dX[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) ss += X[n][e] * X[n][e];
      const float rho = sqrtf(warp_sum(ss) / D + P.rms_eps);
      float dy[E], t = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dy[e] = dx[row[n] * D + lane + 32 * e];
        t += dy[e] * (X[n][e] / rho);
      }
      t = warp_sum(t) / D;
#pragma unroll
      for (int e = 0; e < E; ++e) dX[n][e] = (dy[e] - (X[n][e] / rho) * t) / rho;
    }
    float dqt[NR][W];
    matvec_rs<D, R, NR>(sC, dX, dqt, lane);
    float du[NR][W];
#pragma unroll
    for (int n = 0; n < NR; ++n) features_back<R>(P, tab, ls[n], u[n], dqt[n], du[n], lane);
    float g_[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int e = 0; e < E; ++e) g_[n][e] = 0.f;
    vecmat<D, R, NR>(sP, du, g_, lane);
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      if (lb + n >= l1) break;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dx[row[n] * D + lane + 32 * e] = dX[n][e];
        dq[row[n] * D + lane + 32 * e] = g_[n][e];
      }
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const int m = lane + 32 * w;
        if (m < R) {
          qt_rows[row[n] * R + m] = qt[n][w];
          du_rows[row[n] * R + m] = du[n][w];
        }
      }
    }
  }
}

// Key side, kLrRows tokens of a (batch, head) per warp: recompute U and k~;
// dv = G^T k~, dk~ = G v, dU, dk = dU P_k, where G is the sum of dC over the
// chunks whose prefix state holds the token (its own chunk and every later
// one; dC itself without a window). Writes dU rows for dP_k.
template <int D, int R>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_lr_k_kernel(Problem P, const float2* __restrict__ tab, const uint16_t* __restrict__ k,
                const uint16_t* __restrict__ v, const uint16_t* __restrict__ p_k, const float* __restrict__ dC,
                float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ du_rows, int tok_per_cta) {
  constexpr int E = D / 32, W = (R + 31) / 32, NR = kLrRows;
  extern __shared__ float bwd_smem[];
  float* sP = bwd_smem;           // P_k, fp32 [R][D]
  float* sG = bwd_smem + R * D;   // G of this (batch, head, chunk), fp32 [R][D]
  const int h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int tiles = (P.chunk_tokens + tok_per_cta - 1) / tok_per_cta;
  const int c = blockIdx.x / tiles;
  const size_t bhc = (static_cast<size_t>(b) * P.H + h) * P.n_chunks + c;
  for (int i = threadIdx.x; i < R * D; i += blockDim.x) {
    sP[lane_major<D>(i)] = bf(p_k + i);
    sG[lane_major<D>(i)] = dC[bhc * R * D + i];
  }
  __syncthreads();
  const int l0 = c * P.chunk_tokens + (blockIdx.x % tiles) * tok_per_cta;
  const int l1 = min(chunk_end(P, c), l0 + tok_per_cta);
  for (int lb = l0 + warp * NR; lb < l1; lb += kRowWarps * NR) {
    int ls[NR];
    size_t row[NR];
    float x[NR][E], vv[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      ls[n] = min(lb + n, l1 - 1);
      row[n] = (static_cast<size_t>(b) * P.L + ls[n]) * P.H + h;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[n][e] = bf(k + row[n] * D + lane + 32 * e);
        vv[n][e] = bf(v + row[n] * D + lane + 32 * e);
      }
    }
    float u[NR][W], kt[NR][W];
    matvec_rs<D, R, NR>(sP, x, u, lane);
#pragma unroll
    for (int n = 0; n < NR; ++n) features<R>(P, tab, ls[n], u[n], kt[n], lane);
    float gv[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int e = 0; e < E; ++e) gv[n][e] = 0.f;
    vecmat<D, R, NR>(sG, kt, gv, lane);
    float dkt[NR][W];
    matvec_rs<D, R, NR>(sG, vv, dkt, lane);
    float du[NR][W];
#pragma unroll
    for (int n = 0; n < NR; ++n) features_back<R>(P, tab, ls[n], u[n], dkt[n], du[n], lane);
    float gk[NR][E];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int e = 0; e < E; ++e) gk[n][e] = 0.f;
    vecmat<D, R, NR>(sP, du, gk, lane);
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      if (lb + n >= l1) break;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dv[row[n] * D + lane + 32 * e] = gv[n][e];
        dk[row[n] * D + lane + 32 * e] = gk[n][e];
      }
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const int m = lane + 32 * w;
        if (m < R) du_rows[row[n] * R + m] = du[n][w];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// outer-product sums: out[g] = sum_i A[row(g, i)] (x) B[row(g, i)], M x N
// ---------------------------------------------------------------------------
//
// Group g, item i (i < n_items) maps to the row (g / hg) * n_items * hg + i * hg + g % hg
// of A ([rows, M] fp32) and B ([rows, N], fp32 or bf16): with hg = H and
// n_items = L the groups are the (batch, head) pairs of [B, L, H] rows; with
// hg = 1 and one group, every row. Each CTA sums kOuterRows items in order into
// a partial; the partials are added in chunk order by outer_reduce_kernel.

template <typename TB>
__device__ __forceinline__ float ld_any(const TB* p);
template <>
__device__ __forceinline__ float ld_any<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_any<uint16_t>(const uint16_t* p) { return bf(p); }

template <int M, int N, typename TB>
__global__ void __launch_bounds__(kOuterThreads)
outer_partial_kernel(const float* __restrict__ A, const TB* __restrict__ Bm, int hg, long long n_items,
                     int n_chunks, float* __restrict__ part) {
  // items staged per step: as many as 48 KB of static shared memory holds, up to 64
  constexpr int T = (M + N) * 64 * 4 <= 48 * 1024 ? 64 : 32;
  // thread = output column n and a run of PER consecutive rows m: per item one
  // B value and PER / 4 vector loads of A (the same for the whole warp)
  constexpr int G = kOuterThreads / N;            // row groups
  constexpr int PER = M / G;
  static_assert(G * N == kOuterThreads && PER * G == M && PER % 4 == 0, "outer-product tiling");
  __shared__ __align__(16) float sA[T * M];
  __shared__ float sB[T * N];
  const int g = blockIdx.y, chunk = blockIdx.x;
  const int n = threadIdx.x % N, m0 = (threadIdx.x / N) * PER;
  const long long i0 = static_cast<long long>(chunk) * kOuterRows;
  const long long i1 = min(n_items, i0 + kOuterRows);
  const long long base = static_cast<long long>(g / hg) * n_items * hg + g % hg;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (long long it = i0; it < i1; it += T) {
    const int cnt = static_cast<int>(min(static_cast<long long>(T), i1 - it));
    __syncthreads();
    for (int e = threadIdx.x; e < T * M; e += blockDim.x) {
      const int t = e / M, m = e % M;
      sA[e] = t < cnt ? A[(base + (it + t) * hg) * M + m] : 0.f;
    }
    for (int e = threadIdx.x; e < T * N; e += blockDim.x) {
      const int t = e / N, c = e % N;
      sB[e] = t < cnt ? ld_any<TB>(Bm + (base + (it + t) * hg) * N + c) : 0.f;
    }
    __syncthreads();
    for (int t = 0; t < cnt; ++t) {
      const float bv = sB[t * N + n];
#pragma unroll
      for (int e4 = 0; e4 < PER / 4; ++e4) {
        const float4 a = *reinterpret_cast<const float4*>(sA + t * M + m0 + 4 * e4);
        acc[4 * e4] = fmaf(a.x, bv, acc[4 * e4]);
        acc[4 * e4 + 1] = fmaf(a.y, bv, acc[4 * e4 + 1]);
        acc[4 * e4 + 2] = fmaf(a.z, bv, acc[4 * e4 + 2]);
        acc[4 * e4 + 3] = fmaf(a.w, bv, acc[4 * e4 + 3]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) part[(static_cast<size_t>(g) * n_chunks + chunk) * M * N + (m0 + e) * N + n] = acc[e];
}

// out[g][o] = sum over chunks in order of part[g][chunk][o].
__global__ void outer_reduce_kernel(const float* __restrict__ part, int n_chunks, int mn, float* __restrict__ out) {
  const int g = blockIdx.y;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= mn) return;
  float s = 0.f;
  for (int c = 0; c < n_chunks; ++c) s += part[(static_cast<size_t>(g) * n_chunks + c) * mn + o];
  out[static_cast<size_t>(g) * mn + o] = s;
}

// Causal window: key j sits in the prefix state of its own chunk and of every
// later one, so it receives G_c = sum_{c' >= c} dC_c' (c = its chunk). dC is
// [B][n_chunks][H][R*D] (the order of the outer-product groups), G
// [B][H][n_chunks][R*D]; the sums run from the last chunk down.
__global__ void chunk_suffix_kernel(Problem P, const float* __restrict__ dC, float* __restrict__ G) {
  const size_t rd = static_cast<size_t>(P.rank) * P.d;
  const size_t x = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // (b * H + h) * rd + e
  if (x >= static_cast<size_t>(P.B) * P.H * rd) return;
  const size_t bh = x / rd, e = x % rd;
  const size_t b = bh / P.H, h = bh % P.H;
  float s = 0.f;
  for (int c = P.n_chunks - 1; c >= 0; --c) {
    s += dC[((b * P.n_chunks + c) * P.H + h) * rd + e];
    G[(bh * P.n_chunks + c) * rd + e] = s;
  }
}

// ---------------------------------------------------------------------------
// block-sparse attention: one warp per row, lanes over channels
// ---------------------------------------------------------------------------

// Slot j of a map row: the kept key block; -1 for the padding of a causal
// row (chunks with fewer candidates keep fewer blocks); -2 for an invalid entry.
__device__ __forceinline__ int kept_block(const Problem& P, const int32_t* row, int j) {
  const int kb = __ldg(row + j);
  if (kb >= 0 && kb < P.n_kblk) return kb;
  return (P.causal && kb == -1) ? -1 : -2;
}

// The query block of token l and the end of the keys it sees (chunk_end of its
// chunk; L without a causal window).
__device__ __forceinline__ int token_qblk(const Problem& P, int l, int& hi) {
  const int c = l / P.chunk_tokens;
  hi = chunk_end(P, c);
  return c * P.nq_chunk + (l - c * P.chunk_tokens) / P.block_q;
}

// Per query row: the softmax statistics over its kept keys (lse, in natural
// log units of the scaled score) and D = dO_s . O_s with O_s recomputed in fp32.
template <int D>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_attn_stats_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                      const uint16_t* __restrict__ v, const int32_t* __restrict__ block_idx,
                      const float* __restrict__ do_s, float* __restrict__ lse, float* __restrict__ dd,
                      unsigned* status) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kRowWarps + threadIdx.x / 32;  // (b, l, h)
  if (row >= static_cast<long long>(P.B) * P.L * P.H) return;
  const int h = static_cast<int>(row % P.H);
  const int l = static_cast<int>((row / P.H) % P.L);
  const int b = static_cast<int>(row / (static_cast<long long>(P.H) * P.L));
  int hi;
  const int a = token_qblk(P, l, hi);
  const int32_t* map = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * P.keep;
  const float scale = rsqrtf(static_cast<float>(D));
  float qv[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = bf(q + row * D + lane + 32 * e);
    o[e] = 0.f;
  }
  float m = -INFINITY, s_sum = 0.f;
  bool bad = false;
  for (int j = 0; j < P.keep; ++j) {
    const int kb = kept_block(P, map, j);
    if (kb < 0) {
      bad = bad || kb == -2;
      continue;
    }
    const int t1 = min(hi, (kb + 1) * P.block_k);
    for (int t = kb * P.block_k; t < t1; ++t) {
      const size_t kr = (static_cast<size_t>(b) * P.L + t) * P.H + h;
      float p = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) p += qv[e] * bf(k + kr * D + lane + 32 * e);
      const float s = warp_sum(p) * scale;
      const float mn = fmaxf(m, s);
      const float al = expf(m - mn);  // m = -inf on the first key: 0
      const float w = expf(s - mn);
      s_sum = s_sum * al + w;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = o[e] * al + w * bf(v + kr * D + lane + 32 * e);
      m = mn;
    }
  }
  float dot = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) dot += do_s[row * D + lane + 32 * e] * (s_sum > 0.f ? o[e] / s_sum : 0.f);
  dot = warp_sum(dot);
  if (lane == 0) {
    lse[row] = s_sum > 0.f ? m + logf(s_sum) : INFINITY;  // +inf: no key, every P is 0
    dd[row] = dot;
    if (bad) report_status(status, kStatusBadIndex);
  }
}

// dq += sum over the row's kept keys of P (dO_s . v - D) k / sqrt(d).
template <int D>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_attn_dq_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                   const uint16_t* __restrict__ v, const int32_t* __restrict__ block_idx,
                   const float* __restrict__ do_s, const float* __restrict__ lse, const float* __restrict__ dd,
                   float* __restrict__ dq) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kRowWarps + threadIdx.x / 32;
  if (row >= static_cast<long long>(P.B) * P.L * P.H) return;
  const int h = static_cast<int>(row % P.H);
  const int l = static_cast<int>((row / P.H) % P.L);
  const int b = static_cast<int>(row / (static_cast<long long>(P.H) * P.L));
  int hi;
  const int a = token_qblk(P, l, hi);
  const int32_t* map = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * P.keep;
  const float scale = rsqrtf(static_cast<float>(D));
  const float li = lse[row], di = dd[row];
  float qv[E], gy[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = bf(q + row * D + lane + 32 * e);
    gy[e] = do_s[row * D + lane + 32 * e];
    acc[e] = 0.f;
  }
  for (int j = 0; j < P.keep; ++j) {
    const int kb = kept_block(P, map, j);
    if (kb < 0) continue;
    const int t1 = min(hi, (kb + 1) * P.block_k);
    for (int t = kb * P.block_k; t < t1; ++t) {
      const size_t kr = (static_cast<size_t>(b) * P.L + t) * P.H + h;
      float kk[E], ps = 0.f, pd = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kk[e] = bf(k + kr * D + lane + 32 * e);
        ps += qv[e] * kk[e];
        pd += gy[e] * bf(v + kr * D + lane + 32 * e);
      }
      const float s = warp_sum(ps) * scale;
      const float dp = warp_sum(pd);
      const float ds = expf(s - li) * (dp - di) * scale;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] += ds * kk[e];
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) dq[row * D + lane + 32 * e] += acc[e];
}

// Transposed map: for every (batch, head, key block) the query blocks that
// kept it, ascending. A map row holds distinct key blocks (the selector's
// output) in its kept entries: all keep of them, or keep_of(n_c) for a causal
// row of chunk c (then padded with -1).
__device__ __forceinline__ int row_keep(const Problem& P, int a) {
  return P.causal ? keep_of(P, chunk_cands(P, qblk_chunk(P, a))) : P.keep;
}

// One (batch, head) per CTA: the kept entries are counted per key block with
// shared-memory atomics (the counts do not depend on their order), turned into
// offsets by an exclusive scan, then warp 0 walks the rows in ascending order
// and appends each row index to the lists of the blocks it kept (a row's
// entries are distinct blocks, so no two lanes share a cursor): every list
// comes out ascending. The rows pass through shared memory in chunks.
constexpr int kTmapThreads = 256;
constexpr int kTmapChunkInts = 4096;  // map entries staged per chunk (16 KB)

__global__ void __launch_bounds__(kTmapThreads)
tmap_build_kernel(Problem P, const int32_t* __restrict__ block_idx, int32_t* __restrict__ offs,
                  int32_t* __restrict__ list) {
  extern __shared__ int32_t tmap_smem[];
  const int NK = P.n_kblk;
  int32_t* cur = tmap_smem;                 // [NK + 1]: counts, then offsets, then cursors
  int32_t* rows = tmap_smem + NK + 1;       // [kTmapChunkInts] staged map entries
  const long long bh = blockIdx.x;
  const int32_t* map = block_idx + bh * P.n_qblk * P.keep;
  for (int i = threadIdx.x; i <= NK; i += blockDim.x) cur[i] = 0;
  __syncthreads();
  const long long total = static_cast<long long>(P.n_qblk) * P.keep;
  for (long long e = threadIdx.x; e < total; e += blockDim.x) {
    const int a = static_cast<int>(e / P.keep), j = static_cast<int>(e % P.keep);
    if (j >= row_keep(P, a)) continue;  // -1 padding of a causal row
    const int kb = __ldg(map + e);
    if (kb >= 0 && kb < NK) atomicAdd(&cur[kb + 1], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int kb = 0; kb < NK; ++kb) cur[kb + 1] += cur[kb];
  __syncthreads();
  int32_t* o = offs + bh * (NK + 1);
  for (int i = threadIdx.x; i <= NK; i += blockDim.x) o[i] = cur[i];
  int32_t* out = list + bh * static_cast<long long>(P.n_qblk) * P.keep;
  const int rows_per_chunk = P.keep <= kTmapChunkInts ? kTmapChunkInts / P.keep : 1;
  for (int a0 = 0; a0 < P.n_qblk; a0 += rows_per_chunk) {
    const int a1 = min(P.n_qblk, a0 + rows_per_chunk);
    __syncthreads();  // the previous chunk is consumed (and the offsets are read)
    const int n = (a1 - a0) * P.keep;
    for (int e = threadIdx.x; e < n && e < kTmapChunkInts; e += blockDim.x)
      rows[e] = __ldg(map + static_cast<long long>(a0) * P.keep + e);
    __syncthreads();
    if (threadIdx.x < 32) {
      for (int a = a0; a < a1; ++a) {
        const int ka = row_keep(P, a);
        for (int j = threadIdx.x; j < ka; j += 32) {
          const int kb = (P.keep <= kTmapChunkInts) ? rows[(a - a0) * P.keep + j] : __ldg(map + static_cast<long long>(a) * P.keep + j);
          if (kb >= 0 && kb < NK) out[cur[kb]++] = a;
        }
        __syncwarp();
      }
    }
  }
}

// Per key row: dv += sum_i P_ij dO_s,i and dk += sum_i P_ij (dO_s,i . v_j - D_i) q_i / sqrt(d)
// over the rows i of the query blocks that kept the row's key block, in ascending order.
template <int D>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_attn_dkv_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, const int32_t* __restrict__ offs,
                    const int32_t* __restrict__ list, const float* __restrict__ do_s, const float* __restrict__ lse,
                    const float* __restrict__ dd, float* __restrict__ dk, float* __restrict__ dv) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kRowWarps + threadIdx.x / 32;  // key row (b, t, h)
  if (row >= static_cast<long long>(P.B) * P.L * P.H) return;
  const int h = static_cast<int>(row % P.H);
  const int t = static_cast<int>((row / P.H) % P.L);
  const int b = static_cast<int>(row / (static_cast<long long>(P.H) * P.L));
  const long long bh = static_cast<long long>(b) * P.H + h;
  const int kb = t / P.block_k;
  const float scale = rsqrtf(static_cast<float>(D));
  float kk[E], vv[E], gk[E], gv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kk[e] = bf(k + row * D + lane + 32 * e);
    vv[e] = bf(v + row * D + lane + 32 * e);
    gk[e] = 0.f;
    gv[e] = 0.f;
  }
  const int32_t* o = offs + bh * (P.n_kblk + 1);
  const int32_t* lst = list + bh * static_cast<long long>(P.n_qblk) * P.keep;
  for (int x = o[kb]; x < o[kb + 1]; ++x) {
    const int a = lst[x];
    if (t >= chunk_end(P, qblk_chunk(P, a))) continue;  // past the causal window of the query block
    const int i1 = qblk_end(P, a);
    for (int i = qblk_start(P, a); i < i1; ++i) {
      const size_t qr = (static_cast<size_t>(b) * P.L + i) * P.H + h;
      float qv[E], gy[E], ps = 0.f, pd = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        qv[e] = bf(q + qr * D + lane + 32 * e);
        gy[e] = do_s[qr * D + lane + 32 * e];
        ps += qv[e] * kk[e];
        pd += gy[e] * vv[e];
      }
      const float s = warp_sum(ps) * scale;
      const float dp = warp_sum(pd);
      const float p = expf(s - lse[qr]);
      const float ds = p * (dp - dd[qr]) * scale;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        gv[e] += p * gy[e];
        gk[e] += ds * qv[e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    dk[row * D + lane + 32 * e] += gk[e];
    dv[row * D + lane + 32 * e] += gv[e];
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

constexpr size_t kAlignB = 256;
size_t up(size_t x) { return (x + kAlignB - 1) / kAlignB * kAlignB; }

// Backward scratch, after the forward's workspace regions.
struct BwdLayout {
  size_t o_s, o_lr, do_s, dob, dx, qt, du_q, du_k, lse, dd, dC, G, part, lr_pc, lr_pp, offs, list, total;
  int nch_c, nch_p;  // partial chunks of the dC (per head and causal chunk) and dP (all rows) sums
};

BwdLayout bwd_layout(const Problem& P, size_t base) {
  BwdLayout y{};
  const size_t BH = static_cast<size_t>(P.B) * P.H, rows = BH * P.L;
  const size_t T = rows * P.d, RD = static_cast<size_t>(P.rank) * P.d;
  y.nch_c = (P.chunk_tokens + kOuterRows - 1) / kOuterRows;
  y.nch_p = static_cast<int>((rows + kOuterRows - 1) / kOuterRows);
  size_t off = base;
  y.o_s = off;   off = up(off + T * 2);
  y.o_lr = off;  off = up(off + T * 2);
  y.do_s = off;  off = up(off + (backward_tc_supported(P) ? 0 : T * 4));  // fp32 dO_s: SIMT sparse kernels
  y.dob = off;   off = up(off + (backward_tc_supported(P) ? T * 2 : 0));  // bf16 dO_s for the tensor cores
  y.dx = off;    off = up(off + T * 4);
  // SIMT low-rank path: q~ and dU rows for the outer-product sums; tensor-core
  // path: per-CTA partials of dC and of dP_q / dP_k instead
  const bool lr_tc = lr_tc_supported(P);
  const size_t lr_rows = lr_tc ? 0 : rows;
  y.qt = off;    off = up(off + lr_rows * P.rank * 4);
  y.du_q = off;  off = up(off + lr_rows * P.rank * 4);
  y.du_k = off;  off = up(off + lr_rows * P.rank * 4);
  const size_t lr_parts = lr_tc ? static_cast<size_t>(P.B) * P.n_chunks * P.H * lr_tc_ctas_per_group(P) : 0;
  y.lr_pc = off; off = up(off + lr_parts * RD * 4);
  y.lr_pp = off; off = up(off + lr_parts * RD * 4);
  y.lse = off;   off = up(off + rows * 4);
  y.dd = off;    off = up(off + rows * 4);
  const size_t BHC = BH * P.n_chunks;
  y.dC = off;    off = up(off + BHC * RD * 4);
  y.G = off;     off = up(off + (P.n_chunks > 1 ? BHC * RD * 4 : 0));  // suffix sums over the chunks
  const size_t n_part = lr_tc ? 0
                        : (BHC * y.nch_c > static_cast<size_t>(y.nch_p) ? BHC * y.nch_c : static_cast<size_t>(y.nch_p));
  y.part = off;  off = up(off + n_part * RD * 4);
  y.offs = off;  off = up(off + BH * (P.n_kblk + 1) * 4);
  y.list = off;  off = up(off + BH * P.n_qblk * P.keep * 4);
  y.total = off;
  return y;
}

template <class T>
T* at_(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

template <int R, int N, typename TB>
cudaError_t run_outer(const float* A, const TB* Bm, int hg, long long n_items, int groups, int n_chunks, float* part,
                      float* out, cudaStream_t s) {
  outer_partial_kernel<R, N, TB><<<dim3(n_chunks, groups), kOuterThreads, 0, s>>>(A, Bm, hg, n_items, n_chunks, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  outer_reduce_kernel<<<dim3((R * N + 255) / 256, groups), 256, 0, s>>>(part, n_chunks, R * N, out);
  return cudaGetLastError();
}

template <int D, int R>
cudaError_t run_backward(const Problem& P, const Layout& fy, void* ws, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k, const float* g,
                         const int32_t* block_idx, const uint16_t* d_o, float* dq, float* dk, float* dv, float* dp_q,
                         float* dp_k, float* dg, cudaStream_t s) {
  const BwdLayout y = bwd_layout(P, fy.total);
  unsigned* status = at_<unsigned>(ws, fy.status);
  float2* tab = at_<float2>(ws, fy.rope_tab);
  uint16_t* o_s = at_<uint16_t>(ws, y.o_s);
  uint16_t* o_lr = at_<uint16_t>(ws, y.o_lr);
  float* do_s = at_<float>(ws, y.do_s);
  uint16_t* dob = at_<uint16_t>(ws, y.dob);
  const bool tc_attn = backward_tc_supported(P);
  float* dx = at_<float>(ws, y.dx);
  float* qt = at_<float>(ws, y.qt);
  float* du_q = at_<float>(ws, y.du_q);
  float* du_k = at_<float>(ws, y.du_k);
  float* lse = at_<float>(ws, y.lse);
  float* dd = at_<float>(ws, y.dd);
  float* dC = at_<float>(ws, y.dC);
  float* G = P.n_chunks > 1 ? at_<float>(ws, y.G) : dC;
  float* part = at_<float>(ws, y.part);
  int32_t* offs = at_<int32_t>(ws, y.offs);
  int32_t* list = at_<int32_t>(ws, y.list);
  const long long rows = static_cast<long long>(P.B) * P.L * P.H;
  const unsigned row_ctas = static_cast<unsigned>((rows + kRowWarps - 1) / kRowWarps);
  cudaError_t e;
#define SDA_BWD_TRY(x)             \
  do {                             \
    e = (x);                       \
    if (e != cudaSuccess) return e; \
  } while (0)

  // forward quantities: C (fp32 and bf16 head/tail C^T), O_s, O_lr
  SDA_BWD_TRY(launch_rope_table(P, tab, s));
  SDA_BWD_TRY(launch_lowrank_state(P, fy, tab, k, v, p_k, at_<float>(ws, fy.c_part), at_<float>(ws, fy.c_state),
                                   nullptr, at_<float>(ws, fy.ct_f32), at_<uint16_t>(ws, fy.ct_hi),
                                   at_<uint16_t>(ws, fy.ct_lo), status, true, nullptr, s));
  // tensor-core path: the forward also leaves each row's log2-sum-exp2 for P
  SDA_BWD_TRY(launch_sparse_attn_tc(P, q, k, v, block_idx, o_s, status, s, tc_attn ? lse : nullptr));
  SDA_BWD_TRY(launch_lowrank_readout(P, tab, q, p_q, at_<uint16_t>(ws, fy.ct_hi), at_<uint16_t>(ws, fy.ct_lo), o_lr,
                                     status, true, s));
  // gate
  bwd_gate_kernel<D><<<static_cast<unsigned>((static_cast<long long>(P.B) * P.L + kRowWarps - 1) / kRowWarps),
                       kRowWarps * 32, 0, s>>>(P, o_s, o_lr, g, d_o, tc_attn ? nullptr : do_s, dx, dg,
                                               tc_attn ? dob : nullptr,
                                               tc_attn ? dd : nullptr);
  SDA_BWD_TRY(cudaGetLastError());
  // low-rank branch, query side, then dC and dP_q
  if (lr_tc_supported(P)) {
    // tensor cores: dq, per-CTA partials of dC and dP_q; dC per (batch, chunk, head)
    const int per_group = lr_tc_ctas_per_group(P);
    const int groups = P.B * P.n_chunks * P.H;
    float* pc = at_<float>(ws, y.lr_pc);
    float* pp = at_<float>(ws, y.lr_pp);
    const unsigned rd_blocks = (R * D + 255) / 256;
    // dP sums in two fixed-order levels: per group (into pc, free once dC is formed), then over the groups
    SDA_BWD_TRY(launch_lr_q_tc(P, tab, q, p_q, at_<float>(ws, fy.c_state), dx, dq, pc, pp, status, s));
    outer_reduce_kernel<<<dim3(rd_blocks, groups), 256, 0, s>>>(pc, per_group, R * D, dC);
    SDA_BWD_TRY(cudaGetLastError());
    outer_reduce_kernel<<<dim3(rd_blocks, groups), 256, 0, s>>>(pp, per_group, R * D, pc);
    SDA_BWD_TRY(cudaGetLastError());
    outer_reduce_kernel<<<dim3(rd_blocks, 1), 256, 0, s>>>(pc, groups, R * D, dp_q);
    SDA_BWD_TRY(cudaGetLastError());
    if (P.n_chunks > 1) {
      const size_t n = static_cast<size_t>(P.B) * P.H * R * D;
      chunk_suffix_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(P, dC, G);
      SDA_BWD_TRY(cudaGetLastError());
    }
    // key side: dk, dv and the partials of dP_k
    SDA_BWD_TRY(launch_lr_k_tc(P, tab, k, v, p_k, G, dk, dv, pp, status, s));
    outer_reduce_kernel<<<dim3(rd_blocks, groups), 256, 0, s>>>(pp, per_group, R * D, pc);
    SDA_BWD_TRY(cudaGetLastError());
    outer_reduce_kernel<<<dim3(rd_blocks, 1), 256, 0, s>>>(pc, groups, R * D, dp_k);
    SDA_BWD_TRY(cudaGetLastError());
  } else {
    constexpr int kTokPerCta = 256;
    const size_t lr_smem = 2 * static_cast<size_t>(R) * D * 4;
    const dim3 lr_grid((P.chunk_tokens + kTokPerCta - 1) / kTokPerCta * P.n_chunks, P.H, P.B);
    SDA_BWD_TRY(cudaFuncSetAttribute(bwd_lr_q_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(lr_smem)));
    bwd_lr_q_kernel<D, R><<<lr_grid, kRowWarps * 32, lr_smem, s>>>(P, tab, q, p_q, at_<float>(ws, fy.c_state), dx,
                                                                    dq, qt, du_q, kTokPerCta);
    SDA_BWD_TRY(cudaGetLastError());
    // dC per (batch, causal chunk, head): the rows of the chunk (the whole sequence without a window)
    SDA_BWD_TRY((run_outer<R, D, float>(qt, dx, P.H, P.chunk_tokens, P.B * P.n_chunks * P.H, y.nch_c, part, dC, s)));
    if (P.n_chunks > 1) {
      const size_t n = static_cast<size_t>(P.B) * P.H * R * D;
      chunk_suffix_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(P, dC, G);
      SDA_BWD_TRY(cudaGetLastError());
    }
    SDA_BWD_TRY((run_outer<R, D, uint16_t>(du_q, q, 1, rows, 1, y.nch_p, part, dp_q, s)));
    // key side (state), then dP_k
    SDA_BWD_TRY(cudaFuncSetAttribute(bwd_lr_k_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(lr_smem)));
    bwd_lr_k_kernel<D, R><<<lr_grid, kRowWarps * 32, lr_smem, s>>>(P, tab, k, v, p_k, G, dk, dv, du_k, kTokPerCta);
    SDA_BWD_TRY(cudaGetLastError());
    SDA_BWD_TRY((run_outer<R, D, uint16_t>(du_k, k, 1, rows, 1, y.nch_p, part, dp_k, s)));
  }
  // sparse branch
  if (!tc_attn) {
    bwd_attn_stats_kernel<D><<<row_ctas, kRowWarps * 32, 0, s>>>(P, q, k, v, block_idx, do_s, lse, dd, status);
    SDA_BWD_TRY(cudaGetLastError());
    bwd_attn_dq_kernel<D><<<row_ctas, kRowWarps * 32, 0, s>>>(P, q, k, v, block_idx, do_s, lse, dd, dq);
    SDA_BWD_TRY(cudaGetLastError());
  }
  const size_t tmap_smem = (static_cast<size_t>(P.n_kblk) + 1 + kTmapChunkInts) * 4;
  SDA_BWD_TRY(cudaFuncSetAttribute(tmap_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(tmap_smem)));
  tmap_build_kernel<<<static_cast<unsigned>(P.B * P.H), kTmapThreads, tmap_smem, s>>>(P, block_idx, offs, list);
  SDA_BWD_TRY(cudaGetLastError());
  if (tc_attn) {
    SDA_BWD_TRY(launch_backward_attn_tc(P, q, k, v, dob, block_idx, offs, list, lse, dd, dq, dk, dv, status, s));
  } else {
    bwd_attn_dkv_kernel<D><<<row_ctas, kRowWarps * 32, 0, s>>>(P, q, k, v, offs, list, do_s, lse, dd, dk, dv);
    SDA_BWD_TRY(cudaGetLastError());
  }
#undef SDA_BWD_TRY
  return cudaSuccess;
}

}  // namespace

size_t backward_workspace_bytes(const Problem& P, const Layout& fy) { return bwd_layout(P, fy.total).total; }

cudaError_t launch_backward(const Problem& P, const Layout& fy, void* ws, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k, const float* g,
                            const int32_t* block_idx, const uint16_t* d_o, float* dq, float* dk, float* dv,
                            float* dp_q, float* dp_k, float* dg, cudaStream_t stream) {
#define SDA_BWD_CALL(D_, R_)                                                                                      \
  if (P.d == D_ && P.rank == R_)                                                                                  \
    return run_backward<D_, R_>(P, fy, ws, q, k, v, p_q, p_k, g, block_idx, d_o, dq, dk, dv, dp_q, dp_k, dg, \
                                stream);
  SDA_BWD_CALL(128, 16)
  SDA_BWD_CALL(128, 32)
  SDA_BWD_CALL(128, 64)
  SDA_BWD_CALL(64, 16)
  SDA_BWD_CALL(64, 32)
  SDA_BWD_CALL(64, 64)
#undef SDA_BWD_CALL
  return cudaErrorInvalidValue;
}

}  // namespace sda
