// Low-rank branch of the backward on the tensor cores (d = 128, r = 16 or 32).
//
// Backward of O_lr = RMSNorm(q~^T C), C = sum_j k~_j v_j^T, x~ = R(p) phi(P x)
// (SparkDiffusion summary, robotworld.top, section 2.1; training backpropagates
// through the low-rank branch: H3 portability report, sections 2.1-2.2). Per
// 128-token tile of one (batch, head, causal chunk) every r x d product is a
// tcgen05 MMA with fp32 accumulation in TMEM; the per-row steps (phi and the
// rotation, RMSNorm and its backward, phi' and the inverse rotation) run in
// the four row warps, thread t owning token row t (TMEM lane t).
//
// Query side, per tile (the row's chunk state C, its gradient dO_lr = dy):
//   U = Q P_q^T                 A = Q tile (K-major), B = P_q (K-major)
//   rows: q~ = R phi(U)
//   X = q~ C                    A = q~ head|tail, B = C head|tail (MN-major): 3 products
//   rows: dX = (dy - y mean(dy y)) / rho,  y = X / rho
//   dq~ = dX C^T                A = dX head|tail (K-major), B = C head|tail (K-major): 3 products
//   dC^T += dX^T q~             A = dX (MN-major), B = [q~ head | q~ tail] (MN-major, N = 64)
//   rows: dU = R^T dq~ * phi'(U)
//   dq = dU P_q                 A = dU head|tail (K-major), B = P_q (MN-major): 2 products
//   dP_q^T += Q^T dU            A = Q tile (MN-major), B = [dU head | dU tail] (MN-major)
// Key side, per tile (G = the sum of dC over the chunks whose state holds the key):
//   U = K P_k^T; rows: k~ = R phi(U)
//   dv = k~ G                   A = k~ head|tail, B = G head|tail (MN-major): 3 products
//   dk~ = V G^T                 A = V tile (K-major), B = G head|tail (K-major): 2 products
//   rows: dU = R^T dk~ * phi'(U)
//   dk = dU P_k,  dP_k^T += K^T dU   as on the query side.
// Operands that are not bf16 already (q~, k~, C, G, dX, dU) are split into a
// bf16 head and tail (x = head + tail to ~2^-16) and the products summed, so
// the MMAs carry about fp32 accuracy. dC^T and dP^T accumulate over the CTA's
// tiles in TMEM (both splits of the rank operand side by side, N = 64, added
// at the end) and are written as per-CTA partials, summed in CTA order by the
// outer-product reduce kernel: every sum has a fixed order. dq, dk and dv are
// written here first (the sparse branch adds to them later).
//
// One CTA per run of up to kLrTiles tiles of one (batch, causal chunk, head)
// group; rows past the chunk end are loaded (or zero-filled past L) but take
// zero features and gradients and are not stored. Warps 0-3 are the rows;
// warp 4 allocates TMEM and its lane 0 issues the TMA loads and the MMAs.
// Every wait is bounded (a time-out is reported through the status word).

#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kD = 128;
constexpr int kTile = 128;      // tokens per tile
constexpr int kLrTiles = 8;     // tiles per CTA
constexpr int kThreads = 160;   // 4 row warps + the TMA / MMA warp
constexpr int kTabBytes = 16384;
constexpr int kSlab = kTile * 128;          // [128 rows][128 B], 128-byte swizzle
constexpr int kTileBytes = 2 * kSlab;       // one d = 128 token tile: 2 channel slabs

// TMEM columns: X / dv then dq / dk, U, dq~ / dk~, dC^T, dP^T.
constexpr uint32_t kColX = 0, kColU = 128, kColG = 160, kColDC = 256, kColDP = 320, kColsAlloc = 512;

template <int R>
struct LrSmem {
  static constexpr int kRSlab = R * 128;                  // [R rows][128 B]: 64 channels of an [R][d] matrix
  static constexpr int kA = 0;                            // Q or K tiles, 2 stages
  static constexpr int kV = kA + 2 * kTileBytes;          // key side: V tiles, 2 stages
  static constexpr int kDX = kV;                          // query side: dX head (2 slabs), tail (2 slabs)
  static constexpr int kP = kV + 2 * kTileBytes;          // P_q / P_k: 2 channel slabs
  static constexpr int kM = kP + 2 * kRSlab;              // C or G head (2 slabs) then tail (2 slabs)
  static constexpr int kF = kM + 4 * kRSlab;              // q~ / k~ rows: head ranks at byte 0, tail at 64
  static constexpr int kDU = kF + kSlab;                  // dU rows: head at byte 0, tail at 64
  static constexpr int kTab = kDU + kSlab;
  static constexpr int kBars = kTab + kTabBytes;
  static constexpr int kTotal = kBars + 256;
};

enum {
  LB_AFULL = 0, LB_AEMPTY = 2, LB_VFULL = 4, LB_MREADY = 6, LB_UFULL, LB_FFULL, LB_XFULL, LB_DXFULL, LB_GFULL,
  LB_DUFULL, LB_OFULL, LB_OREAD, LB_DONE, LB_N
};

// Arrivals per phase: 1 for the TMA and MMA completions, 128 for the rows.
__device__ __forceinline__ void init_lr_barriers(uint64_t* bars) {
  for (int i = 0; i < LB_N; ++i) {
    const bool rows = i == LB_MREADY || i == LB_FFULL || i == LB_DXFULL || i == LB_DUFULL || i == LB_OREAD;
    tc::mbar_init(&bars[i], rows ? 128 : 1);
  }
}

// phi = elu + 1 and its derivative, with the fast exponential (as the forward's feature kernels)
__device__ __forceinline__ float elu1(float u) { return u > 0.f ? u + 1.f : __expf(u); }
__device__ __forceinline__ float elu1_prime(float u) { return u > 0.f ? 1.f : __expf(u); }

// x = head + tail, both bf16 (round to nearest), as the low halves of two words.
__device__ __forceinline__ void split2(float x, uint32_t& head, uint32_t& tail) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  head = __bfloat16_as_ushort(h);
  tail = __bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(h)));
}

// The CTA's work: group g = (b * n_chunks + c) * H + h, tiles [t0, t1) of the chunk.
struct LrWork {
  int b, h, c, g, l0, t0, n_tiles, rows_in_chunk;
};
__device__ __forceinline__ LrWork lr_work(const Problem& P, int per_group) {
  LrWork w;
  w.g = blockIdx.x / per_group;
  const int j = blockIdx.x % per_group;
  w.h = w.g % P.H;
  w.c = (w.g / P.H) % P.n_chunks;
  w.b = w.g / (P.H * P.n_chunks);
  const int tiles = (P.chunk_tokens + kTile - 1) / kTile;
  w.t0 = j * kLrTiles;
  w.n_tiles = min(kLrTiles, tiles - w.t0);
  w.l0 = w.c * P.chunk_tokens;
  w.rows_in_chunk = P.chunk_tokens;
  return w;
}

// [R][d] fp32 (C or G of one group) into bf16 head / tail slabs: element (m, c)
// at row m, channel c of slab c / 64 (K-major for N = m, MN-major for K = m).
template <int R>
__device__ __forceinline__ void stage_rd_split(const float* __restrict__ src, unsigned char* dst, int t128) {
  using S = LrSmem<R>;
  for (int e = t128; e < R * (kD / 8); e += 128) {
    const int m = e / (kD / 8), c8 = e % (kD / 8);
    const float4 a = __ldg(reinterpret_cast<const float4*>(src + m * kD + 8 * c8));
    const float4 bq = __ldg(reinterpret_cast<const float4*>(src + m * kD + 8 * c8 + 4));
    const float v[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
    uint32_t hd[8], tl[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) split2(v[i], hd[i], tl[i]);
    const uint32_t off = (c8 / 8) * S::kRSlab + tc::sw128_offset(m, c8 % 8);
    *reinterpret_cast<uint4*>(dst + off) =
        make_uint4(hd[0] | hd[1] << 16, hd[2] | hd[3] << 16, hd[4] | hd[5] << 16, hd[6] | hd[7] << 16);
    *reinterpret_cast<uint4*>(dst + 2 * S::kRSlab + off) =
        make_uint4(tl[0] | tl[1] << 16, tl[2] | tl[3] << 16, tl[4] | tl[5] << 16, tl[6] | tl[7] << 16);
  }
}

// P ([R][d] bf16) into two channel slabs, same layout.
template <int R>
__device__ __forceinline__ void stage_p(const uint16_t* __restrict__ p, unsigned char* dst, int t128) {
  using S = LrSmem<R>;
  for (int e = t128; e < R * (kD / 8); e += 128) {
    const int m = e / (kD / 8), c8 = e % (kD / 8);
    *reinterpret_cast<uint4*>(dst + (c8 / 8) * S::kRSlab + tc::sw128_offset(m, c8 % 8)) =
        __ldg(reinterpret_cast<const uint4*>(p + m * kD) + c8);
  }
}

// R fp32 values of the row (rank order) as its rank row: head ranks in the
// 16-byte chunks 0..R/8-1, tail ranks in chunks 4..4+R/8-1 of a K-major row.
template <int R>
__device__ __forceinline__ void put_rank_row(unsigned char* slab, int row, const float (&x)[R]) {
  uint32_t hd[R], tl[R];
#pragma unroll
  for (int m = 0; m < R; ++m) split2(x[m], hd[m], tl[m]);
#pragma unroll
  for (int c = 0; c < R / 8; ++c) {
    *reinterpret_cast<uint4*>(slab + tc::sw128_offset(row, c)) =
        make_uint4(hd[8 * c] | hd[8 * c + 1] << 16, hd[8 * c + 2] | hd[8 * c + 3] << 16,
                   hd[8 * c + 4] | hd[8 * c + 5] << 16, hd[8 * c + 6] | hd[8 * c + 7] << 16);
    *reinterpret_cast<uint4*>(slab + tc::sw128_offset(row, 4 + c)) =
        make_uint4(tl[8 * c] | tl[8 * c + 1] << 16, tl[8 * c + 2] | tl[8 * c + 3] << 16,
                   tl[8 * c + 4] | tl[8 * c + 5] << 16, tl[8 * c + 6] | tl[8 * c + 7] << 16);
  }
}

// cos / sin of the rotation pairs of token l, from the staged table.
struct RowRope {
  const float2* t;
  const float2* h;
  const float2* w;
  int pt, ph;
  __device__ __forceinline__ float2 at(int mm) const { return mm < pt ? t[mm] : (mm < pt + ph ? h[mm] : w[mm]); }
};
__device__ __forceinline__ RowRope row_rope(const Problem& P, const float2* tab, int l) {
  const int gw = l % P.grid_w, gh = (l / P.grid_w) % P.grid_h, gt = l / (P.grid_w * P.grid_h);
  RowRope r;
  r.t = tab + gt * P.pairs_t;
  r.h = tab + P.grid_t * P.pairs_t + gh * P.pairs_h - P.pairs_t;
  r.w = tab + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + gw * P.pairs_w - P.pairs_t - P.pairs_h;
  r.pt = P.pairs_t;
  r.ph = P.pairs_h;
  return r;
}

template <int R>
__device__ __forceinline__ void load_cols(uint32_t taddr, float (&x)[R]) {
  uint32_t u[R];
#pragma unroll
  for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(taddr + 16 * c, u + 16 * c);
  tc::tmem_wait_ld();
#pragma unroll
  for (int m = 0; m < R; ++m) x[m] = __uint_as_float(u[m]);
}

// x~ = R phi(u) (zero for rows that are not stored).
template <int R>
__device__ __forceinline__ void features(const float (&u)[R], const RowRope& rr, bool valid, float (&f)[R]) {
#pragma unroll
  for (int mm = 0; mm < R / 2; ++mm) {
    const float xx = elu1(u[2 * mm]), yy = elu1(u[2 * mm + 1]);
    const float2 cs = rr.at(mm);
    f[2 * mm] = valid ? xx * cs.x - yy * cs.y : 0.f;
    f[2 * mm + 1] = valid ? xx * cs.y + yy * cs.x : 0.f;
  }
}

// dU = R^T g * phi'(u) (the transpose of a rotation by a turns by -a).
template <int R>
__device__ __forceinline__ void features_back(const float (&u)[R], const float (&g)[R], const RowRope& rr, bool valid,
                                              float (&du)[R]) {
#pragma unroll
  for (int mm = 0; mm < R / 2; ++mm) {
    const float2 cs = rr.at(mm);
    const float a = g[2 * mm], b = g[2 * mm + 1];
    du[2 * mm] = valid ? (a * cs.x + b * cs.y) * elu1_prime(u[2 * mm]) : 0.f;
    du[2 * mm + 1] = valid ? (b * cs.x - a * cs.y) * elu1_prime(u[2 * mm + 1]) : 0.f;
  }
}

// The row's 128 TMEM columns (fp32) into a [128 rows][128] fp32 staging tile
// (float4 j of row t at position j ^ (t % 32): a warp's lanes spread over the
// banks), then, after the row warps synchronise, each warp writes 32 whole rows
// with one coalesced 512-byte store per row. Rows that are not stored are
// skipped. Every lane runs the TMEM loads (warp-collective).
__device__ __forceinline__ void store_rows_staged(uint32_t taddr, float* stage, int t, float* dst_base,
                                                  size_t row_stride, int my_off, int n_valid) {
  float4* st4 = reinterpret_cast<float4*>(stage);
#pragma unroll 1
  for (int c = 0; c < kD / 32; ++c) {
    uint32_t r[32];
    tc::tmem_ld32(taddr + 32 * c, r);
    tc::tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int j = 8 * c + k;
      st4[t * 32 + (j ^ (t & 31))] = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                                 __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
    }
  }
  tc::named_barrier(1, 128);
  const int lane = t & 31, w = t >> 5;
  for (int i = 0; i < 32; ++i) {
    const int rt = 32 * w + i;  // tile row
    if (rt >= n_valid) break;  // warp-uniform
    const int j = lane ^ (rt & 31);
    const int off = __shfl_sync(0xffffffffu, my_off, i);  // global row of tile row rt (lane i's row)
    reinterpret_cast<float4*>(dst_base + static_cast<size_t>(off) * row_stride)[j] = st4[rt * 32 + lane];
  }
  tc::named_barrier(1, 128);  // the staging tile is free again
}

// The same through a 16 KB staging slab, 32 channels at a time: per round
// every thread puts its row's 32 values (float4 j of row t at j ^ (t % 8)),
// the row warps synchronise, and each warp writes its 32 rows, eight lanes
// per 128-byte row piece (four rows per store instruction).
__device__ __forceinline__ void store_rows_chunked(uint32_t taddr, float* stage, int t, float* dst_base,
                                                   size_t row_stride, int my_off, int n_valid) {
  float4* st4 = reinterpret_cast<float4*>(stage);
  const int lane = t & 31, w = t >> 5;
#pragma unroll 1
  for (int c = 0; c < kD / 32; ++c) {
    uint32_t r[32];
    tc::tmem_ld32(taddr + 32 * c, r);
    tc::tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k)
      st4[t * 8 + (k ^ (t & 7))] = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                               __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
    tc::named_barrier(1, 128);
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const int rt = 32 * w + i + lane / 8;  // tile row of this lane's piece
      const int k = lane % 8;                // its float4 within the 32 channels
      const int off = __shfl_sync(0xffffffffu, my_off, i + lane / 8);
      if (rt < n_valid)
        reinterpret_cast<float4*>(dst_base + static_cast<size_t>(off) * row_stride + 32 * c)[k] =
            st4[rt * 8 + (k ^ (rt & 7))];
    }
    tc::named_barrier(1, 128);  // the staging slab is free for the next round
  }
}

// dC^T / dP^T partial of the CTA: lane = channel c; columns m (head) and 32 + m
// (tail) of the N = 64 accumulator add up to element (m, c); written [m][c].
template <int R>
__device__ __forceinline__ void write_partial(uint32_t taddr, float* dst, int c) {
  uint32_t r[64];
  tc::tmem_ld32p(taddr, r);
  tc::tmem_ld32p(taddr + 32, r + 32);
  tc::tmem_wait_ld();
#pragma unroll
  for (int m = 0; m < R; ++m) dst[m * kD + c] = __uint_as_float(r[m]) + __uint_as_float(r[32 + m]);
}

// One K-major MMA chain over the d = 128 channels: D (+)= A[128 x 128] B^T, A in
// two 64-channel slabs of 128 rows, B in two slabs of n_rows rows.
__device__ __forceinline__ void mma_kmajor_d(uint32_t d, const unsigned char* a, const unsigned char* b, int b_slab,
                                             uint32_t idesc, bool acc) {
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const int hf = kk / 4, c = kk % 4;
    tc::mma_ss(d, tc::smem_desc_sw128(a + hf * kSlab + c * 32, 16, 1024),
               tc::smem_desc_sw128(b + hf * b_slab + c * 32, 16, 1024), idesc, (acc || kk > 0) ? 1u : 0u);
  }
}

// D (+)= A[128 x r] B with A a rank row slab (K-major: head at byte 0, tail at 64)
// and B an [R][d] head or tail pair of slabs given MN-major (K = rank rows, N = d).
template <int R>
__device__ __forceinline__ void mma_rank_k(uint32_t d, const unsigned char* a, int a_part, const unsigned char* b,
                                           uint32_t idesc, bool acc) {
  using S = LrSmem<R>;
#pragma unroll
  for (int kk = 0; kk < R / 16; ++kk)
    tc::mma_ss(d, tc::smem_desc_sw128(a + 64 * a_part + 32 * kk, 16, 1024),
               tc::smem_desc_sw128(b + kk * 16 * 128, S::kRSlab, 1024), idesc, (acc || kk > 0) ? 1u : 0u);
}

// D^T[d x 64] (+)= A^T B over the 128 rows of a tile: A a [rows][d] tile of two
// channel slabs and B a rank row slab (N = 64: head | tail), both MN-major.
__device__ __forceinline__ void mma_outer(uint32_t d, const unsigned char* a, const unsigned char* b, uint32_t idesc,
                                          bool acc) {
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    tc::mma_ss(d, tc::smem_desc_sw128(a + kk * 16 * 128, kSlab, 1024), tc::smem_desc_sw128(b + kk * 16 * 128, kSlab, 1024),
               idesc, (acc || kk > 0) ? 1u : 0u);
}

// ---------------------------------------------------------------------------
// query side
// ---------------------------------------------------------------------------

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
bwd_lrq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, Problem P, const float2* __restrict__ tab,
                  const uint16_t* __restrict__ p_q, const float* __restrict__ c_state, const float* __restrict__ dy,
                  float* __restrict__ dq, float* __restrict__ part_c, float* __restrict__ part_p, int per_group,
                  unsigned* status) {
  using S = LrSmem<R>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * LB_N);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * LB_N + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const LrWork w = lr_work(P, per_group);
  const int tab_n = rope_table_entries(P);
  const bool tab_smem = tab_n * 8 <= kTabBytes;

  if (threadIdx.x == 0) {
    init_lr_barriers(bars);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 4) {
    tc::tmem_alloc(tmem_slot, kColsAlloc);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA + MMA
      volatile int never = 0;
      constexpr uint32_t id_u = tc::idesc_bf16(128, R, false);          // A, B K-major
      constexpr uint32_t id_x = tc::idesc_bf16(128, kD, true);          // B MN-major
      constexpr uint32_t id_g = tc::idesc_bf16(128, R, false);
      constexpr uint32_t id_o = tc::idesc_bf16(128, 64, true) | (1u << 15);  // A and B MN-major
      auto load_tile = [&](int i) {
        const int s = i & 1;
        tc::mbar_arrive_expect_tx(&bars[LB_AFULL + s], kTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          tc::tma_load_4d(smem + S::kA + s * kTileBytes + hf * kSlab, &tm_q, &bars[LB_AFULL + s], 64 * hf, w.h,
                          w.l0 + (w.t0 + i) * kTile, w.b);
      };
      load_tile(0);
      int issued = 1;
      bool ok = tc::wait1(&bars[LB_MREADY], 0, abort_flag);
      if (ok) tc::fence_after_sync();
      const unsigned char* mh = smem + S::kM;
      const unsigned char* mt = smem + S::kM + 2 * S::kRSlab;
      for (int i = 0; i < w.n_tiles && ok; ++i) {
        const int s = i & 1;
        const unsigned char* a = smem + S::kA + s * kTileBytes;
        ok = tc::wait1(&bars[LB_AFULL + s], (i >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_kmajor_d(tmem + kColU, a, smem + S::kP, S::kRSlab, id_u, false);  // U = Q P_q^T
        tc::commit(&bars[LB_UFULL]);
        if (i + 1 < w.n_tiles) {  // next tile into the other stage, once tile i - 1's dP MMA is done with it
          if (i >= 1) ok = tc::wait1(&bars[LB_AEMPTY + (s ^ 1)], ((i - 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          load_tile(i + 1);
          ++issued;
        }
        // X = q~ C (3 products), once the rows wrote q~ and read the previous dq
        ok = tc::wait1(&bars[LB_FFULL], i & 1, abort_flag);
        if (ok && i >= 1) ok = tc::wait1(&bars[LB_OREAD], (i - 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 0, mh, id_x, false);
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 0, mt, id_x, true);
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 1, mh, id_x, true);
        tc::commit(&bars[LB_XFULL]);
        // dq~ = dX C^T (3 products) and dC^T += dX^T [q~ head | q~ tail]
        ok = tc::wait1(&bars[LB_DXFULL], i & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const unsigned char* dxh = smem + S::kDX;
        const unsigned char* dxt = smem + S::kDX + 2 * kSlab;
        mma_kmajor_d(tmem + kColG, dxh, mh, S::kRSlab, id_g, false);
        mma_kmajor_d(tmem + kColG, dxh, mt, S::kRSlab, id_g, true);
        mma_kmajor_d(tmem + kColG, dxt, mh, S::kRSlab, id_g, true);
        mma_outer(tmem + kColDC, dxh, smem + S::kF, id_o, i > 0);
        mma_outer(tmem + kColDC, dxt, smem + S::kF, id_o, true);
        tc::commit(&bars[LB_GFULL]);
        // dq = dU P_q (2 products) and dP_q^T += Q^T [dU head | dU tail]
        ok = tc::wait1(&bars[LB_DUFULL], i & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_rank_k<R>(tmem + kColX, smem + S::kDU, 0, smem + S::kP, id_x, false);
        mma_rank_k<R>(tmem + kColX, smem + S::kDU, 1, smem + S::kP, id_x, true);
        mma_outer(tmem + kColDP, a, smem + S::kDU, id_o, i > 0);
        tc::commit(&bars[LB_OFULL]);
        tc::commit(&bars[LB_AEMPTY + s]);
      }
      tc::commit(&bars[LB_DONE]);
      tc::wait1(&bars[LB_DONE], 0, &never);
      for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
        tc::wait1(&bars[LB_AFULL + (j & 1)], (j >> 1) & 1, &never);
    }
  } else {
    // ------------------------------------------------------------ rows
    const int t = threadIdx.x;  // row of the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    float2* stab = reinterpret_cast<float2*>(smem + S::kTab);
    stage_p<R>(p_q, smem + S::kP, t);
    stage_rd_split<R>(c_state + (static_cast<size_t>(w.b * P.H + w.h) * P.n_chunks + w.c) * R * kD, smem + S::kM, t);
    if (tab_smem)
      for (int e = t; e < tab_n; e += 128) stab[e] = __ldg(tab + e);
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars[LB_MREADY]);
    tc::named_barrier(1, 128);
    const float2* rt = tab_smem ? stab : tab;
    bool ok = true;
    for (int i = 0; i < w.n_tiles && ok; ++i) {
      const int lt = (w.t0 + i) * kTile + t;  // token within the chunk
      const bool valid = lt < w.rows_in_chunk && w.l0 + lt < P.L;
      const int l = valid ? w.l0 + lt : w.l0;
      const size_t row = (static_cast<size_t>(w.b) * P.L + l) * P.H + w.h;
      const RowRope rr = row_rope(P, rt, l);
      // the row's dO_lr (512 bytes) toward L2 while U, q~ and X are formed
      if (valid)
        for (int c = 0; c < kD * 4; c += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(dy + row * kD + c / 4));
      // q~
      ok = tc::wait_warp(&bars[LB_UFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      float u[R], f[R];
      load_cols<R>(tmem + lane_base + kColU, u);
      features<R>(u, rr, valid, f);
      put_rank_row<R>(smem + S::kF, t, f);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_FFULL]);
      // dX: pass 1 the sums, pass 2 the values (head, tail into the dX slabs)
      ok = tc::wait_warp(&bars[LB_XFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      const float* dyr = dy + row * kD;
      float ss = 0.f, sd = 0.f;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + lane_base + kColX + 32 * c, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 g4 = __ldg(reinterpret_cast<const float4*>(dyr + 32 * c) + k);
          const float x0 = __uint_as_float(r[4 * k]), x1 = __uint_as_float(r[4 * k + 1]);
          const float x2 = __uint_as_float(r[4 * k + 2]), x3 = __uint_as_float(r[4 * k + 3]);
          ss += x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
          sd += g4.x * x0 + g4.y * x1 + g4.z * x2 + g4.w * x3;
        }
      }
      const float rho = sqrtf(ss / kD + P.rms_eps);
      const float inv_rho = 1.f / rho;
      const float tm = sd * inv_rho / kD;  // mean(dy y), y = X / rho
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + lane_base + kColX + 32 * c, r);
        tc::tmem_wait_ld();
        unsigned char* sh = smem + S::kDX + (c / 2) * kSlab;
        unsigned char* st = sh + 2 * kSlab;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(dyr + 32 * c + 8 * k));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(dyr + 32 * c + 8 * k + 4));
          const float gy[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          uint32_t hd[8], tl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = __uint_as_float(r[8 * k + e]);
            split2(valid ? (gy[e] - x * inv_rho * tm) * inv_rho : 0.f, hd[e], tl[e]);
          }
          const uint32_t off = tc::sw128_offset(t, 4 * (c % 2) + k);
          *reinterpret_cast<uint4*>(sh + off) =
              make_uint4(hd[0] | hd[1] << 16, hd[2] | hd[3] << 16, hd[4] | hd[5] << 16, hd[6] | hd[7] << 16);
          *reinterpret_cast<uint4*>(st + off) =
              make_uint4(tl[0] | tl[1] << 16, tl[2] | tl[3] << 16, tl[4] | tl[5] << 16, tl[6] | tl[7] << 16);
        }
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_DXFULL]);
      // dU
      ok = tc::wait_warp(&bars[LB_GFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      float g[R], du[R];
      load_cols<R>(tmem + lane_base + kColU, u);
      load_cols<R>(tmem + lane_base + kColG, g);
      features_back<R>(u, g, rr, valid, du);
      put_rank_row<R>(smem + S::kDU, t, du);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_DUFULL]);
      // dq
      ok = tc::wait_warp(&bars[LB_OFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      {
        // the tile's valid rows are its first n_valid (rows past the chunk end or L come last);
        // warp w stores tile rows 32w .. 32w + 31, whose global row offsets it gathers by shuffle
        const int n_valid = min(kTile, min(w.rows_in_chunk, P.L - w.l0) - (w.t0 + i) * kTile);
        store_rows_staged(tmem + lane_base + kColX, reinterpret_cast<float*>(smem + S::kDX), t, dq, kD,
                          static_cast<int>(row), n_valid);
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_OREAD]);
    }
    if (ok) ok = tc::wait_warp(&bars[LB_DONE], 0, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      const size_t slot = static_cast<size_t>(blockIdx.x);  // = g * per_group + j
      write_partial<R>(tmem + lane_base + kColDC, part_c + slot * R * kD, t);
      write_partial<R>(tmem + lane_base + kColDP, part_p + slot * R * kD, t);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) report_status(status, kStatusTimeout);
  if (warp == 4) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kColsAlloc);
  }
}

// ---------------------------------------------------------------------------
// key side
// ---------------------------------------------------------------------------

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
bwd_lrk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Problem P,
                  const float2* __restrict__ tab, const uint16_t* __restrict__ p_k, const float* __restrict__ gsum,
                  float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ part_p, int per_group,
                  unsigned* status) {
  using S = LrSmem<R>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * LB_N);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * LB_N + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const LrWork w = lr_work(P, per_group);
  const int tab_n = rope_table_entries(P);
  const bool tab_smem = tab_n * 8 <= kTabBytes;

  if (threadIdx.x == 0) {
    init_lr_barriers(bars);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 4) {
    tc::tmem_alloc(tmem_slot, kColsAlloc);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA + MMA
      volatile int never = 0;
      constexpr uint32_t id_u = tc::idesc_bf16(128, R, false);
      constexpr uint32_t id_x = tc::idesc_bf16(128, kD, true);
      constexpr uint32_t id_g = tc::idesc_bf16(128, R, false);
      constexpr uint32_t id_o = tc::idesc_bf16(128, 64, true) | (1u << 15);
      auto load_tile = [&](int i) {
        const int s = i & 1;
        const int l = w.l0 + (w.t0 + i) * kTile;
        tc::mbar_arrive_expect_tx(&bars[LB_AFULL + s], kTileBytes);
        tc::mbar_arrive_expect_tx(&bars[LB_VFULL + s], kTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
          tc::tma_load_4d(smem + S::kA + s * kTileBytes + hf * kSlab, &tm_k, &bars[LB_AFULL + s], 64 * hf, w.h, l,
                          w.b);
          tc::tma_load_4d(smem + S::kV + s * kTileBytes + hf * kSlab, &tm_v, &bars[LB_VFULL + s], 64 * hf, w.h, l,
                          w.b);
        }
      };
      load_tile(0);
      int issued = 1;
      bool ok = tc::wait1(&bars[LB_MREADY], 0, abort_flag);
      if (ok) tc::fence_after_sync();
      const unsigned char* mh = smem + S::kM;
      const unsigned char* mt = smem + S::kM + 2 * S::kRSlab;
      for (int i = 0; i < w.n_tiles && ok; ++i) {
        const int s = i & 1;
        const unsigned char* a = smem + S::kA + s * kTileBytes;
        const unsigned char* vt = smem + S::kV + s * kTileBytes;
        ok = tc::wait1(&bars[LB_AFULL + s], (i >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_kmajor_d(tmem + kColU, a, smem + S::kP, S::kRSlab, id_u, false);  // U = K P_k^T
        tc::commit(&bars[LB_UFULL]);
        if (i + 1 < w.n_tiles) {
          if (i >= 1) ok = tc::wait1(&bars[LB_AEMPTY + (s ^ 1)], ((i - 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          load_tile(i + 1);
          ++issued;
        }
        // dv = k~ G (3 products) and dk~ = V G^T (2 products), once the rows wrote
        // k~ and read the previous dk
        ok = tc::wait1(&bars[LB_FFULL], i & 1, abort_flag);
        if (ok) ok = tc::wait1(&bars[LB_VFULL + s], (i >> 1) & 1, abort_flag);
        if (ok && i >= 1) ok = tc::wait1(&bars[LB_OREAD], (i - 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 0, mh, id_x, false);
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 0, mt, id_x, true);
        mma_rank_k<R>(tmem + kColX, smem + S::kF, 1, mh, id_x, true);
        mma_kmajor_d(tmem + kColG, vt, mh, S::kRSlab, id_g, false);
        mma_kmajor_d(tmem + kColG, vt, mt, S::kRSlab, id_g, true);
        tc::commit(&bars[LB_GFULL]);
        // dk = dU P_k (2 products) and dP_k^T += K^T [dU head | dU tail], once the
        // rows wrote dU (after reading dv)
        ok = tc::wait1(&bars[LB_DUFULL], i & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        mma_rank_k<R>(tmem + kColX, smem + S::kDU, 0, smem + S::kP, id_x, false);
        mma_rank_k<R>(tmem + kColX, smem + S::kDU, 1, smem + S::kP, id_x, true);
        mma_outer(tmem + kColDP, a, smem + S::kDU, id_o, i > 0);
        tc::commit(&bars[LB_OFULL]);
        tc::commit(&bars[LB_AEMPTY + s]);
      }
      tc::commit(&bars[LB_DONE]);
      tc::wait1(&bars[LB_DONE], 0, &never);
      for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j) {
        tc::wait1(&bars[LB_AFULL + (j & 1)], (j >> 1) & 1, &never);
        tc::wait1(&bars[LB_VFULL + (j & 1)], (j >> 1) & 1, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int t = threadIdx.x;
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    float2* stab = reinterpret_cast<float2*>(smem + S::kTab);
    stage_p<R>(p_k, smem + S::kP, t);
    stage_rd_split<R>(gsum + (static_cast<size_t>(w.b * P.H + w.h) * P.n_chunks + w.c) * R * kD, smem + S::kM, t);
    if (tab_smem)
      for (int e = t; e < tab_n; e += 128) stab[e] = __ldg(tab + e);
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars[LB_MREADY]);
    tc::named_barrier(1, 128);
    const float2* rt = tab_smem ? stab : tab;
    bool ok = true;
    for (int i = 0; i < w.n_tiles && ok; ++i) {
      const int lt = (w.t0 + i) * kTile + t;
      const bool valid = lt < w.rows_in_chunk && w.l0 + lt < P.L;
      const int l = valid ? w.l0 + lt : w.l0;
      const size_t row = (static_cast<size_t>(w.b) * P.L + l) * P.H + w.h;
      const RowRope rr = row_rope(P, rt, l);
      // k~
      ok = tc::wait_warp(&bars[LB_UFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      float u[R], f[R];
      load_cols<R>(tmem + lane_base + kColU, u);
      features<R>(u, rr, valid, f);
      put_rank_row<R>(smem + S::kF, t, f);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_FFULL]);
      // dv, then dU
      ok = tc::wait_warp(&bars[LB_GFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      // the tile's valid rows are its first n_valid; warp w gathers the global offsets of its 32 rows
      const int n_valid = min(kTile, min(w.rows_in_chunk, P.L - w.l0) - (w.t0 + i) * kTile);
      // dv through the feature slab (the dv MMA that read k~ is complete)
      store_rows_chunked(tmem + lane_base + kColX, reinterpret_cast<float*>(smem + S::kF), t, dv, kD,
                         static_cast<int>(row), n_valid);
      float g[R], du[R];
      load_cols<R>(tmem + lane_base + kColG, g);
      features_back<R>(u, g, rr, valid, du);
      put_rank_row<R>(smem + S::kDU, t, du);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_DUFULL]);
      // dk
      ok = tc::wait_warp(&bars[LB_OFULL], i & 1, abort_flag);
      if (tc::named_barrier_or(1, 128, !ok)) { ok = false; break; }  // the row warps leave together
      tc::fence_after_sync();
      // dk through the feature slab again (the next tile's features come after)
      store_rows_chunked(tmem + lane_base + kColX, reinterpret_cast<float*>(smem + S::kF), t, dk, kD,
                         static_cast<int>(row), n_valid);
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[LB_OREAD]);
    }
    if (ok) ok = tc::wait_warp(&bars[LB_DONE], 0, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      write_partial<R>(tmem + lane_base + kColDP, part_p + static_cast<size_t>(blockIdx.x) * R * kD, t);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) report_status(status, kStatusTimeout);
  if (warp == 4) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kColsAlloc);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, L, H, d] bf16; box = 64 channels x 1 head x 128 tokens x 1 batch (zero fill past L).
bool make_tile_map(CUtensorMap* map, const void* base, const Problem& P) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(P.d), static_cast<cuuint64_t>(P.H),
                              static_cast<cuuint64_t>(P.L), static_cast<cuuint64_t>(P.B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(P.d) * 2, static_cast<cuuint64_t>(P.H) * P.d * 2,
                                 static_cast<cuuint64_t>(P.L) * P.H * P.d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kTile), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R>
cudaError_t run_lrq(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q, const float* c_state,
                    const float* dy, float* dq, float* part_c, float* part_p, unsigned* status, cudaStream_t s) {
  CUtensorMap mq;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  if (!make_tile_map(&mq, q, P)) return cudaErrorInvalidValue;
  const int smem = LrSmem<R>::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_lrq_tc_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int per_group = lr_tc_ctas_per_group(P);
  const long long grid = static_cast<long long>(P.B) * P.n_chunks * P.H * per_group;
  bwd_lrq_tc_kernel<R><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(mq, P, tab, p_q, c_state, dy, dq, part_c,
                                                                            part_p, per_group, status);
  return cudaGetLastError();
}

template <int R>
cudaError_t run_lrk(const Problem& P, const float2* tab, const uint16_t* k, const uint16_t* v, const uint16_t* p_k,
                    const float* gsum, float* dk, float* dv, float* part_p, unsigned* status, cudaStream_t s) {
  CUtensorMap mk, mv;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  if (!make_tile_map(&mk, k, P) || !make_tile_map(&mv, v, P)) return cudaErrorInvalidValue;
  const int smem = LrSmem<R>::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_lrk_tc_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int per_group = lr_tc_ctas_per_group(P);
  const long long grid = static_cast<long long>(P.B) * P.n_chunks * P.H * per_group;
  bwd_lrk_tc_kernel<R><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(mk, mv, P, tab, p_k, gsum, dk, dv, part_p,
                                                                            per_group, status);
  return cudaGetLastError();
}

}  // namespace

bool lr_tc_supported(const Problem& P) { return P.d == kD && (P.rank == 16 || P.rank == 32); }

int lr_tc_ctas_per_group(const Problem& P) {
  const int tiles = (P.chunk_tokens + kTile - 1) / kTile;
  return (tiles + kLrTiles - 1) / kLrTiles;
}

cudaError_t launch_lr_q_tc(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                           const float* c_state, const float* dy, float* dq, float* part_c, float* part_p,
                           unsigned* status, cudaStream_t s) {
  if (P.rank == 16) return run_lrq<16>(P, tab, q, p_q, c_state, dy, dq, part_c, part_p, status, s);
  if (P.rank == 32) return run_lrq<32>(P, tab, q, p_q, c_state, dy, dq, part_c, part_p, status, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_lr_k_tc(const Problem& P, const float2* tab, const uint16_t* k, const uint16_t* v,
                           const uint16_t* p_k, const float* gsum, float* dk, float* dv, float* part_p,
                           unsigned* status, cudaStream_t s) {
  if (P.rank == 16) return run_lrk<16>(P, tab, k, v, p_k, gsum, dk, dv, part_p, status, s);
  if (P.rank == 32) return run_lrk<32>(P, tab, k, v, p_k, gsum, dk, dv, part_p, status, s);
  return cudaErrorInvalidValue;
}

}  // namespace sda
