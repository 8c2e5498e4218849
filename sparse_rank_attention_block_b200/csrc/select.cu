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
// tokens in order, so the fp32 result does not depend on scheduling. Each mean
// is stored as a bf16 head plus a bf16 tail (x ~= head + tail to ~2^-17),
// with the channels of a row permuted into the register order of the
// m16n8k16 MMA fragments, so the score kernel loads its fragments with
// 16-byte loads and no shared-memory staging.
//
// Kernel 2 (score + select): one CTA per (batch, head, 16 or 32 query
// blocks). Scores of those rows against every key block run on the tensor
// cores as head*head + head*tail + tail*head (fp32 accumulation, fixed order:
// a relative error ~2^-17 per product, far inside the 1e-4 top-k boundary gap
// the parity tests guarantee) into shared memory; then each warp radix-selects
// the k-th largest score of its rows (4 passes of 8 bits over an
// order-preserving uint32 key) and compacts the winners in ascending index
// order with ballots.

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kPoolMaxThreads = 640;
constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kSmemLimit = 232448;
constexpr int kChunkKeys = 64;  // pooled keys per shared-memory ring slot

// Position of channel c in a permuted row of d channels: lane t of a quad
// holds, for every 16-channel k-step ks, the pairs (16ks + 2t, +1) and
// (16ks + 8 + 2t, +1) as 4 consecutive elements of its d/4-element slice.
__host__ __device__ __forceinline__ int frag_pos(int c, int d) {
  const int ks = c / 16, hh = (c / 8) & 1, t = (c % 8) / 2, e = c & 1;
  return t * (d / 4) + ks * 4 + hh * 2 + e;
}

__global__ void __launch_bounds__(kPoolMaxThreads)
pool_kernel(Problem P, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
            uint16_t* __restrict__ q_mean, uint16_t* __restrict__ k_mean) {
  const int per_b = P.n_qblk + P.n_kblk;
  const int b = blockIdx.x / per_b;
  const int j = blockIdx.x % per_b;
  const bool is_q = j < P.n_qblk;
  const uint16_t* src = is_q ? q : k;
  const int blk = is_q ? P.block_q : P.block_k;
  const int n = is_q ? j : j - P.n_qblk;
  const int N = is_q ? P.n_qblk : P.n_kblk;
  uint16_t* dst = is_q ? q_mean : k_mean;  // rows of [head: d][tail: d] bf16, permuted
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
    uint16_t* row = dst + ((static_cast<size_t>(b) * P.H + h) * N + n) * 2 * P.d;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float h0, t0, h1, t1;
      split_bf16(acc[2 * t] * inv, h0, t0);
      split_bf16(acc[2 * t + 1] * inv, h1, t1);
      const int pos = frag_pos(c0 + 2 * t, P.d);
      *reinterpret_cast<uint32_t*>(row + pos) = pack_bf16(h0, h1);
      *reinterpret_cast<uint32_t*>(row + P.d + pos) = pack_bf16(t0, t1);
    }
  }
}

// Larger float <=> larger key; -0 is folded onto +0 first so equal scores tie.
__device__ __forceinline__ uint32_t order_key(float s) {
  if (s == 0.0f) s = 0.0f;
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Load the d/4-element slices (head and tail) of one permuted row as 32-bit words.
template <int D>
__device__ __forceinline__ void load_frag_row(const uint16_t* row, int t, bool ok, uint32_t (&hi)[D / 8],
                                              uint32_t (&lo)[D / 8]) {
  if (ok) {
    const uint4* ph = reinterpret_cast<const uint4*>(row + t * (D / 4));
    const uint4* pl = reinterpret_cast<const uint4*>(row + D + t * (D / 4));
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const uint4 x = __ldg(ph + i), y = __ldg(pl + i);
      hi[4 * i] = x.x; hi[4 * i + 1] = x.y; hi[4 * i + 2] = x.z; hi[4 * i + 3] = x.w;
      lo[4 * i] = y.x; lo[4 * i + 1] = y.y; lo[4 * i + 2] = y.z; lo[4 * i + 3] = y.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < D / 8; ++i) hi[i] = lo[i] = 0u;
  }
}

// Top-k of one row of NK scores by one warp, scores in registers (lane holds
// indices lane, lane + 32, ...). First a bisection on the score value that
// stops as soon as exactly k scores lie at or above the threshold (that set
// is then the answer: no score ties at the boundary); if the bracket
// collapses first (a tie at the k-th place), the k-th largest order key T is
// found bit by bit. Winners are written in ascending index order, keys equal
// to T taken from the lowest index up.
__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

template <int MAXPER>
__device__ __forceinline__ void select_row_reg(const float* row, int NK, int keep, int32_t* out, int lane) {
  float v[MAXPER];
  float vmin = INFINITY, vmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    const int c = 32 * i + lane;
    const float x = c < NK ? row[c] : -INFINITY;  // padding: below every finite threshold
    v[i] = x;
    if (c < NK) {
      vmin = fminf(vmin, x);
      vmax = fmaxf(vmax, x);
    }
  }
  vmin = warp_min(vmin);
  vmax = warp_max(vmax);
  auto count_ge = [&](float t) {
    int c0 = 0, c1 = 0;
#pragma unroll
    for (int i = 0; i < MAXPER; i += 2) {
      c0 += v[i] >= t;
      if (i + 1 < MAXPER) c1 += v[i + 1] >= t;
    }
    return static_cast<int>(__reduce_add_sync(0xffffffffu, c0 + c1));
  };
  // count(v >= lo) >= keep and count(v >= hi) < keep throughout
  float lo = vmin, hi = INFINITY, thr = 0.f;
  bool exact = keep == NK;  // every score kept
  if (exact) thr = vmin;
  if (!exact && vmax > vmin) {
    hi = vmax;
    if (count_ge(hi) >= keep) {  // the top keys all equal vmax: a tie, leave it to the key search
      hi = INFINITY;
    } else {
      for (int it = 0; it < 40; ++it) {
        const float mid = lo + 0.5f * (hi - lo);
        if (!(mid > lo && mid < hi)) break;
        const int c = count_ge(mid);
        if (c == keep) {
          thr = mid;
          exact = true;
          break;
        }
        if (c > keep) lo = mid;
        else hi = mid;
      }
    }
  }
  const unsigned lt = (1u << lane) - 1u;
  if (exact) {
    int taken = 0;
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
      if (32 * i >= NK) break;
      const unsigned tb = __ballot_sync(0xffffffffu, v[i] >= thr);
      const int pos = taken + __popc(tb & lt);
      if (v[i] >= thr && pos < keep) out[pos] = 32 * i + lane;
      taken += __popc(tb);
    }
    return;
  }
  // tie at the k-th place: exact search over the order keys (padding key 0 is never a candidate)
  uint32_t kk[MAXPER];
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    const bool in = 32 * i + lane < NK;
    kk[i] = in ? order_key(v[i]) : 0u;
    if (in) {
      kmin = min(kmin, kk[i]);
      kmax = max(kmax, kk[i]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const uint32_t diff = kmin ^ kmax;
  const int bits = diff ? 32 - __clz(diff) : 0;
  uint32_t T = bits == 32 ? 0u : (kmin & ~((1u << bits) - 1u));  // common prefix: count(key >= T) = NK
  for (int bit = bits - 1; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int c0 = 0;
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) c0 += kk[i] >= cand;
    if (static_cast<int>(__reduce_add_sync(0xffffffffu, c0)) >= keep) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) gt += kk[i] > T;
  const int remaining = keep - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));  // ties of T to take
  int taken = 0, ties = 0;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    if (32 * i >= NK) break;
    const bool g = kk[i] > T, e = kk[i] == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, e);
    const bool take = g || (e && ties + __popc(eqb & lt) < remaining);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = taken + __popc(tb & lt);
    if (take && pos < keep) out[pos] = 32 * i + lane;
    taken += __popc(tb);
    ties += __popc(eqb);
  }
}

template <int D, int ROWS>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_select_kernel(Problem P, const uint16_t* __restrict__ q_mean, const uint16_t* __restrict__ k_mean,
                    int32_t* __restrict__ block_idx, unsigned* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int MT = ROWS / 16;
  constexpr int kRowBytes = 2 * D * 2;                                      // one pooled row: head + tail bf16
  const int NK = P.n_kblk;
  unsigned char* ring = smem;                                               // [2][kChunkKeys rows]
  float* sc = reinterpret_cast<float*>(smem + 2 * kChunkKeys * kRowBytes);  // [ROWS][NK]
  uint32_t* hist = reinterpret_cast<uint32_t*>(sc + ROWS * NK);             // [warps][256]
  __shared__ uint64_t bars[4];                                              // full[2], empty[2]
  __shared__ int abort_s;

  const int a0 = blockIdx.x * ROWS;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * P.H + h;
  const int tid = threadIdx.x;
  const int warp = tid / 32;
  const int lane = tid % 32;
  const int g = lane / 4, t = lane % 4;
  volatile int* abort_flag = &abort_s;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[s], 1);
      tc::mbar_init(&bars[2 + s], kScoreWarps);
    }
    abort_s = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();

  // ---- phase 1: scores on the tensor cores ----
  // The pooled keys of this head stream through a 2-slot shared-memory ring
  // in chunks of kChunkKeys rows (bulk copies issued by thread 0); warp w
  // scores the w-th 8-key tile of every chunk against the ROWS query rows.
  uint32_t ahi[MT][D / 16][4], alo[MT][D / 16][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    uint32_t h0[D / 8], l0[D / 8], h1[D / 8], l1[D / 8];
    const int r0 = a0 + 16 * mt + g, r1 = r0 + 8;
    load_frag_row<D>(q_mean + (bh * P.n_qblk + r0) * 2 * D, t, r0 < P.n_qblk, h0, l0);
    load_frag_row<D>(q_mean + (bh * P.n_qblk + r1) * 2 * D, t, r1 < P.n_qblk, h1, l1);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      ahi[mt][ks][0] = h0[2 * ks]; ahi[mt][ks][1] = h1[2 * ks];
      ahi[mt][ks][2] = h0[2 * ks + 1]; ahi[mt][ks][3] = h1[2 * ks + 1];
      alo[mt][ks][0] = l0[2 * ks]; alo[mt][ks][1] = l1[2 * ks];
      alo[mt][ks][2] = l0[2 * ks + 1]; alo[mt][ks][3] = l1[2 * ks + 1];
    }
  }
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(k_mean + bh * NK * 2 * D);
  const int n_chunks = (NK + kChunkKeys - 1) / kChunkKeys;
  auto issue = [&](int c) {
    const int rows = min(kChunkKeys, NK - c * kChunkKeys);
    const uint32_t bytes = static_cast<uint32_t>(rows * kRowBytes);
    tc::mbar_arrive_expect_tx(&bars[c & 1], bytes);
    tc::bulk_load(ring + (c & 1) * kChunkKeys * kRowBytes, kbase + static_cast<size_t>(c) * kChunkKeys * kRowBytes,
                  bytes, &bars[c & 1]);
  };
  int issued = 0;
  if (tid == 0) {
    issue(0);
    issued = 1;
  }
  bool ok = true;
  for (int c = 0; c < n_chunks && ok; ++c) {
    if (tid == 0 && c + 1 < n_chunks) {
      // slot (c + 1) & 1 is free once every warp has finished chunk c - 1
      if (c >= 1) ok = tc::wait1(&bars[2 + ((c + 1) & 1)], ((c - 1) >> 1) & 1, abort_flag);
      if (ok) {
        issue(c + 1);
        issued = c + 2;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;  // warp 0 follows thread 0's verdict
    if (!ok) break;
    ok = tc::wait_warp(&bars[c & 1], (c >> 1) & 1, abort_flag);
    if (!ok) break;
    const unsigned char* slot = ring + (c & 1) * kChunkKeys * kRowBytes;
    const int key0 = c * kChunkKeys + 8 * warp;  // first key of this warp's tile
    if (key0 < NK) {
      uint32_t chi[D / 8], clo[D / 8];
      const uint4* ph = reinterpret_cast<const uint4*>(slot + (8 * warp + g) * kRowBytes + t * (D / 4) * 2);
      const uint4* pl = reinterpret_cast<const uint4*>(slot + (8 * warp + g) * kRowBytes + D * 2 + t * (D / 4) * 2);
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const uint4 x = ph[i], y = pl[i];
        chi[4 * i] = x.x; chi[4 * i + 1] = x.y; chi[4 * i + 2] = x.z; chi[4 * i + 3] = x.w;
        clo[4 * i] = y.x; clo[4 * i + 1] = y.y; clo[4 * i + 2] = y.z; clo[4 * i + 3] = y.w;
      }
      float acc[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          mma_bf16_16816(acc[mt], ahi[mt][ks], chi[2 * ks], chi[2 * ks + 1]);
          mma_bf16_16816(acc[mt], ahi[mt][ks], clo[2 * ks], clo[2 * ks + 1]);
          mma_bf16_16816(acc[mt], alo[mt][ks], chi[2 * ks], chi[2 * ks + 1]);
        }
      }
      const int key = key0 + 2 * t;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        float* r0 = sc + (16 * mt + g) * NK;
        float* r1 = sc + (16 * mt + g + 8) * NK;
        if (key < NK) {
          r0[key] = acc[mt][0];
          r1[key] = acc[mt][2];
        }
        if (key + 1 < NK) {
          r0[key + 1] = acc[mt][1];
          r1[key + 1] = acc[mt][3];
        }
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&bars[2 + (c & 1)]);
  }
  if (tid == 0) {
    // drain: every bulk copy issued has landed before the ring is reused or freed
    volatile int never = 0;
    for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c) tc::wait1(&bars[c & 1], (c >> 1) & 1, &never);
  }
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) report_status(status, kStatusTimeout);
    return;
  }

  // ---- phase 2: per-row selection + ascending compaction ----
  uint32_t* hw = hist + warp * 256;
  const int keep = P.keep;
  if (NK <= 32 * 64) {
    // keys in registers
    for (int rr = warp; rr < ROWS; rr += kScoreWarps) {
      const int a = a0 + rr;
      if (a >= P.n_qblk) break;
      int32_t* out = block_idx + (bh * P.n_qblk + a) * keep;
      const float* row = sc + rr * NK;
      if (NK <= 32 * 8) select_row_reg<8>(row, NK, keep, out, lane);
      else if (NK <= 32 * 20) select_row_reg<20>(row, NK, keep, out, lane);
      else if (NK <= 32 * 40) select_row_reg<40>(row, NK, keep, out, lane);
      else select_row_reg<64>(row, NK, keep, out, lane);
    }
    return;
  }
  // longer rows: 8-bit radix passes over a shared-memory histogram
  for (int rr = warp; rr < ROWS; rr += kScoreWarps) {
    const int a = a0 + rr;
    if (a >= P.n_qblk) break;
    const float* row = sc + rr * NK;
    // Bits shared by every key of the row need no pass: start the radix
    // digits below the common prefix of the smallest and largest key (pooled
    // scores share sign and exponent, which would pile every key into one bin).
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int c = lane; c < NK; c += 32) {
      const uint32_t u = order_key(row[c]);
      kmin = min(kmin, u);
      kmax = max(kmax, u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    const uint32_t diff = kmin ^ kmax;
    int bits = diff ? 32 - __clz(diff) : 0;  // low bits still undecided
    uint32_t pmask = bits == 32 ? 0u : ~((1u << bits) - 1u);
    uint32_t prefix = kmin & pmask;
    int remaining = keep;
    while (bits > 0) {
      const int width = bits < 8 ? bits : 8;
      const int shift = bits - width;
      const uint32_t dmask = (1u << width) - 1u;
#pragma unroll
      for (int e = 0; e < 8; ++e) hw[lane * 8 + e] = 0;
      __syncwarp();
      for (int c = lane; c < NK; c += 32) {
        const uint32_t u = order_key(row[c]);
        if ((u & pmask) == prefix) atomicAdd(&hw[(u >> shift) & dmask], 1u);
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
      pmask |= dmask << shift;
      bits = shift;
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
    __syncwarp();
  }
}

// Shared memory of the score kernel: key ring, ROWS score rows, radix histograms.
size_t score_smem(const Problem& P, int rows) {
  return static_cast<size_t>(2) * kChunkKeys * 4 * P.d + static_cast<size_t>(rows) * P.n_kblk * 4 +
         kScoreWarps * 256 * 4;
}

int score_rows(const Problem& P) { return score_smem(P, 32) <= static_cast<size_t>(kSmemLimit) ? 32 : 16; }

template <int D, int ROWS>
cudaError_t run_score(const Problem& P, const uint16_t* q_mean, const uint16_t* k_mean, int32_t* block_idx,
                      unsigned* status, cudaStream_t stream) {
  const size_t smem = score_smem(P, ROWS);
  cudaError_t e = cudaFuncSetAttribute(score_select_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((P.n_qblk + ROWS - 1) / ROWS, P.H, P.B);
  score_select_kernel<D, ROWS><<<grid, kScoreThreads, smem, stream>>>(P, q_mean, k_mean, block_idx, status);
  return cudaGetLastError();
}

}  // namespace

size_t score_select_smem_bytes(const Problem& P) { return score_smem(P, score_rows(P)); }

cudaError_t launch_block_select(const Problem& P, const uint16_t* q, const uint16_t* k, uint16_t* q_mean,
                                uint16_t* k_mean, int32_t* block_idx, unsigned* status, cudaStream_t stream) {
  const int threads = (P.H * P.d / 8) < kPoolMaxThreads ? (P.H * P.d / 8) : kPoolMaxThreads;
  pool_kernel<<<P.B * (P.n_qblk + P.n_kblk), threads, 0, stream>>>(P, q, k, q_mean, k_mean);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = score_rows(P);
  if (P.d == 128) return rows == 32 ? run_score<128, 32>(P, q_mean, k_mean, block_idx, status, stream)
                                    : run_score<128, 16>(P, q_mean, k_mean, block_idx, status, stream);
  return rows == 32 ? run_score<64, 32>(P, q_mean, k_mean, block_idx, status, stream)
                    : run_score<64, 16>(P, q_mean, k_mean, block_idx, status, stream);
}

}  // namespace sda
