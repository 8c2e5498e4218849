// Low-rank state C = sum_j k~_j v_j^T on the tcgen05 tensor cores (d = 128,
// and d = 64 with two heads per tile) (SparkDiffusion summary, robotworld.top,
// section 2.1: features and global state equations).
//
// d = 64: a work item covers the heads 2p and 2p + 1 (a head past H reads as
// zeros and writes nothing), whose 64 channels fill the two 64-channel slabs
// of a d = 128 tile, so every MMA keeps M = 128: U = K [P_k 0; 0 P_k]^T gives
// both heads' U side by side (N = 2r), the features of both heads stand in
// one B operand (N = 4r: head 2p head|tail, head 2p+1 head|tail) and channel
// rows 0..63 of C^T read the first half of the accumulator, rows 64..127 the
// second.
//
// Persistent: one CTA per SM walks work items (batch, head, piece of 256..2048 tokens)
// in a fixed round-robin order; each item leaves one r x d partial state. With
// a causal window the pieces tile each chunk on its own (the last one of a
// chunk ends at the chunk end, its last tile ragged: rows past it take zero
// features), so the fixed-order reduce can form every chunk's prefix state.
// A single thread keeps about one tcgen05.mma in flight, so the two MMA
// streams of a 128-token tile issue from separate warps:
//   warp 0      TMA of the K tiles (128 tokens x d, 128-byte swizzle) into a
//               2-stage ring, freed as soon as U is computed;
//   warp 1      TMEM owner; U = K P_k^T (M=128 tokens, N=r, K=d) into the U
//               buffer of the tile's parity;
//   warp 2      TMA of the V tiles into a 3-stage ring (2 for r = 64), freed
//               by the state MMA;
//   warp 3      C^T += V^T [k~_head | k~_tail] (M=d, N=2r, K=128 tokens; A =
//               V read MN-major, B = the features from shared memory): one
//               MMA chain carries both bf16 parts, summed at the readout;
//   warps 4..7  features of the even tiles: one thread per token, phi and the
//               rank-truncated 3D RoPE on its U row, k~ split into a bf16
//               head and tail written K-major into shared memory; they also
//               read each finished partial state out of TMEM (thread = channel);
//   warps 8..11 features of the odd tiles.
// With r <= 32 and a k_mean output, the kernel also yields the selector's
// block means of K (so the selector reads only Q): per tile, warp 1 issues
// Kbar^T = K^T [1_block0 | 1_block1] (M=d, N=16, K=128 tokens; A = the K tile
// read MN-major, B = a constant 0/1 block-membership tile), and the tile's
// feature group turns the two fp32 sums into bf16 head+tail means.
// The accumulator is double-buffered across items, U, the features and the
// block sums across tiles. All waits are bounded (2 s) and report through the
// status word.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kThreads = 384;  // 12 warps
constexpr int kKStages = 2;
constexpr int kMaxVStages = 3;
// V ring depth: 3 tiles where shared memory allows (r <= 32), else 2
template <int R>
constexpr int v_stages() { return R <= 32 ? 3 : 2; }
constexpr int kTileTok = 128;
constexpr int kChunkTok = 2048;   // tokens per work item (partial state), at most
constexpr int kChunkMin = 256;
constexpr int kItemsWanted = 4 * 148;  // work items that keep a B200's SMs evenly busy (a tuning figure)
constexpr int kTabBytes = 16384;  // RoPE table staged in shared memory when it fits

// PAIR: d = 64, two heads per tile. NU = U columns per tile, NF = feature rows.
template <int R, bool PAIR>
struct StateSmem {
  static constexpr int NU = PAIR ? 2 * R : R;
  static constexpr int NF = 2 * NU;                            // head | tail of every rank column
  static constexpr int kVSt = PAIR ? 2 : v_stages<R>();
  static constexpr int kTabB = PAIR ? 8192 : kTabBytes;
  static constexpr int kTileBytes = 2 * kTileTok * 128;        // one tile: 2 slabs x 128 rows x 128 B
  static constexpr int kKtBytes = 2 * NF * 128;                // 2 token slabs x NF rows x 128 B
  static constexpr int kKRing = 0;                             // kKStages K tiles
  static constexpr int kVRing = kKRing + kKStages * kTileBytes;      // kVSt V tiles
  static constexpr int kKt = kVRing + kVSt * kTileBytes;       // 2 buffers
  static constexpr int kPk = kKt + 2 * kKtBytes;               // P_k: 2 channel slabs x NU rows x 128 B
  static constexpr int kTab = kPk + 2 * NU * 128;
  static constexpr bool kPool = R <= 32;                       // room for the block-sum tile
  static constexpr int kInd = kTab + kTabB;                    // 0/1 membership: 2 token slabs x 16 rows x 128 B
  static constexpr int kBars = kInd + (kPool ? 2 * 16 * 128 : 0);
  static constexpr int kTotal = kBars + 256;
};

enum {
  SB_KFULL = 0, SB_KEMPTY = 2, SB_VFULL = 4, SB_VEMPTY = 4 + kMaxVStages, SB_UFULL = 4 + 2 * kMaxVStages,
  SB_UFREE = SB_UFULL + 2, SB_KTFULL = SB_UFREE + 2, SB_KTEMPTY = SB_KTFULL + 2, SB_CDONE = SB_KTEMPTY + 2,
  SB_CFREE = SB_CDONE + 2, SB_PKREADY = SB_CFREE + 2, SB_TABREADY = SB_PKREADY + 1, SB_PFULL = SB_TABREADY + 1,
  SB_PFREE = SB_PFULL + 2, SB_DRAIN = SB_PFREE + 2, SB_N = SB_DRAIN + 2
};

struct Item {
  int bh, chunk, l0, l1, n_tiles;  // chunk: the piece's index among the (batch, head)'s n_split partials
};

// Piece p of a (batch, head): piece p % n_sub of causal chunk p / n_sub (the
// whole sequence is one chunk without a window). With head pairs, bh numbers
// (batch, head pair).
__device__ __forceinline__ Item item_of(const Problem& P, int n_split, int n_sub, int chunk_tok, int it) {
  Item x;
  x.bh = it / n_split;
  x.chunk = it % n_split;
  const int c = x.chunk / n_sub;
  x.l0 = c * P.chunk_tokens + (x.chunk % n_sub) * chunk_tok;
  x.l1 = min(min(P.L, chunk_end(P, c)), x.l0 + chunk_tok);
  x.n_tiles = (x.l1 - x.l0 + kTileTok - 1) / kTileTok;
  return x;
}

// phi(u) = elu(u) + 1 with the fast exponential, and x split into a bf16 head
// (rounded half up) and a bf16 tail, both as raw 16-bit patterns: integer
// work, off the quarter-rate conversion pipe.
__device__ __forceinline__ float elu1_fast(float u) { return u > 0.f ? u + 1.f : __expf(u); }
__device__ __forceinline__ void split_bits(float x, uint32_t& head, uint32_t& tail) {
  const uint32_t hb = (__float_as_uint(x) + 0x8000u) & 0xffff0000u;
  head = hb >> 16;
  tail = (__float_as_uint(x - __uint_as_float(hb)) + 0x8000u) >> 16;
}

template <int R, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
lowrank_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        Problem P, int n_chunks, int n_sub, int chunk_tok, const float2* __restrict__ tab,
                        const uint16_t* __restrict__ p_k,
                        float* __restrict__ c_part, uint16_t* __restrict__ k_mean, unsigned* status) {
  constexpr int D = PAIR ? 64 : 128;     // channels of one head
  using S = StateSmem<R, PAIR>;
  constexpr int NU = S::NU, NF = S::NF;
  constexpr int kVStages = S::kVSt;
  const int HP = PAIR ? (P.H + 1) / 2 : P.H;  // (head pairs of) heads per batch
  // U0, U1 (NU), C0, C1 (NF), block sums P0, P1 (16 each, pooled form)
  constexpr int kUsed = 2 * NU + 2 * NF + (S::kPool ? 32 : 0);
  constexpr uint32_t kCols = (kUsed <= 128) ? 128 : ((kUsed <= 256) ? 256 : 512);
  const bool pool = S::kPool && k_mean != nullptr;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * SB_N);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * SB_N + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_items = P.B * HP * n_chunks;
  const int tab_n = rope_table_entries(P);
  const bool tab_smem = tab_n * 8 <= S::kTabB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kVStages; ++s) {
      tc::mbar_init(&bars[SB_VFULL + s], 1);
      tc::mbar_init(&bars[SB_VEMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[SB_KFULL + s], 1);
      tc::mbar_init(&bars[SB_KEMPTY + s], 1);
      tc::mbar_init(&bars[SB_UFULL + s], 1);
      tc::mbar_init(&bars[SB_UFREE + s], 128);
      tc::mbar_init(&bars[SB_KTFULL + s], 128);
      tc::mbar_init(&bars[SB_KTEMPTY + s], 1);
      tc::mbar_init(&bars[SB_CDONE + s], 1);
      tc::mbar_init(&bars[SB_CFREE + s], 128);
      tc::mbar_init(&bars[SB_PFULL + s], 1);
      tc::mbar_init(&bars[SB_PFREE + s], 128);
      tc::mbar_init(&bars[SB_DRAIN + s], 1);
    }
    tc::mbar_init(&bars[SB_PKREADY], 128);
    tc::mbar_init(&bars[SB_TABREADY], 128);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto colU = [](int ub) { return static_cast<uint32_t>(ub * NU); };
  auto colC = [](int cb) { return static_cast<uint32_t>(2 * NU + cb * NF); };
  auto colP = [](int pb) { return static_cast<uint32_t>(2 * NU + 2 * NF + pb * 16); };

  if (warp < 4) {
    if (lane == 0) {
      volatile int never = 0;
      if (warp == 0 || warp == 2) {
        // ---------------------------------------------------------- producers (K: warp 0, V: warp 2)
        const bool is_k = warp == 0;
        const int nst = is_k ? kKStages : kVStages;
        uint64_t* full = &bars[is_k ? SB_KFULL : SB_VFULL];
        uint64_t* empty = &bars[is_k ? SB_KEMPTY : SB_VEMPTY];
        unsigned char* ring = smem + (is_k ? S::kKRing : S::kVRing);
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
        bool ok = true;
        int gi = 0;  // tiles issued by this CTA
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
          const Item x = item_of(P, n_chunks, n_sub, chunk_tok, it);
          const int b = x.bh / HP, h = x.bh % HP;
          for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
            const int st = gi % nst;
            ok = tc::wait1(&empty[st], ((gi / nst) & 1) ^ 1, abort_flag);
            if (!ok) break;
            unsigned char* dst = ring + st * S::kTileBytes;
            tc::mbar_arrive_expect_tx(&full[st], S::kTileBytes);
            const int l0 = x.l0 + t * kTileTok;
            // slab hf: channels 64 hf.. of head h, or (pairs) head 2h + hf (zero fill past H)
            for (int hf = 0; hf < 2; ++hf)
              tc::tma_load_4d(dst + hf * kTileTok * 128, map, &full[st], PAIR ? 0 : 64 * hf, PAIR ? 2 * h + hf : h, l0, b);
          }
        }
        for (int j = gi - nst < 0 ? 0 : gi - nst; j < gi; ++j) tc::wait1(&full[j % nst], (j / nst) & 1, &never);
      } else if (warp == 1) {
        // ---------------------------------------------------------- U issuer
        constexpr uint32_t idesc_u = tc::idesc_bf16(128, NU, false);
        bool ok = tc::wait1(&bars[SB_PKREADY], 0, abort_flag);
        if (ok) tc::fence_after_sync();
        int gi = 0;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
          const Item x = item_of(P, n_chunks, n_sub, chunk_tok, it);
          for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
            const int st = gi % kKStages, ub = gi & 1;
            ok = tc::wait1(&bars[SB_KFULL + st], (gi / kKStages) & 1, abort_flag);
            // U[ub] is free once the features of tile gi - 2 have read it
            if (ok && gi >= 2) ok = tc::wait1(&bars[SB_UFREE + ub], ((gi >> 1) - 1) & 1, abort_flag);
            if (!ok) break;
            tc::fence_after_sync();
            const unsigned char* kt = smem + S::kKRing + st * S::kTileBytes;
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk) {
              const int hf = kk / 4, c = kk % 4;
              const uint64_t da = tc::smem_desc_sw128(kt + hf * kTileTok * 128 + c * 32, 16, 1024);
              const uint64_t db = tc::smem_desc_sw128(smem + S::kPk + hf * NU * 128 + c * 32, 16, 1024);
              tc::mma_ss(tmem + colU(ub), da, db, idesc_u, kk > 0 ? 1u : 0u);
            }
            tc::commit(&bars[SB_UFULL + ub]);
            if (pool) {
              // block sums of K over the tile's two 64-token blocks (buffer free once
              // the feature group has read the sums of tile gi - 2)
              if (gi >= 2) ok = tc::wait1(&bars[SB_PFREE + ub], ((gi >> 1) - 1) & 1, abort_flag);
              if (!ok) break;
              constexpr uint32_t idesc_p = tc::idesc_bf16(128, 16, false) | (1u << 15);
#pragma unroll
              for (int kk = 0; kk < kTileTok / 16; ++kk) {
                const uint64_t da = tc::smem_desc_sw128(kt + kk * 16 * 128, kTileTok * 128, 1024);
                const uint64_t db = tc::smem_desc_sw128(smem + S::kInd + (kk / 4) * 16 * 128 + (kk % 4) * 32, 16, 1024);
                tc::mma_ss(tmem + colP(ub), da, db, idesc_p, kk > 0 ? 1u : 0u);
              }
              tc::commit(&bars[SB_PFULL + ub]);
            }
            tc::commit(&bars[SB_KEMPTY + st]);
          }
        }
        tc::commit(&bars[SB_DRAIN]);
        tc::wait1(&bars[SB_DRAIN], 0, &never);
      } else {
        // ---------------------------------------------------------- C issuer
        // C^T[cb] (+)= V^T [k~_head | k~_tail]: A = V (d contiguous: MN-major), B = features (K-major)
        constexpr uint32_t idesc_c = tc::idesc_bf16(128, NF, false) | (1u << 15);
        bool ok = true;
        int gi = 0, ii = 0;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ii) {
          const Item x = item_of(P, n_chunks, n_sub, chunk_tok, it);
          const int cb = ii & 1;
          for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
            const int ub = gi & 1, vs = gi % kVStages;
            ok = tc::wait1(&bars[SB_KTFULL + ub], (gi >> 1) & 1, abort_flag);
            if (ok) ok = tc::wait1(&bars[SB_VFULL + vs], (gi / kVStages) & 1, abort_flag);
            // the accumulator is free once the readout of item ii - 2 has read it
            if (ok && t == 0) ok = tc::wait1(&bars[SB_CFREE + cb], ((ii >> 1) & 1) ^ 1, abort_flag);
            if (!ok) break;
            tc::fence_after_sync();
            const unsigned char* vt = smem + S::kVRing + vs * S::kTileBytes;
            const unsigned char* ft = smem + S::kKt + ub * S::kKtBytes;
#pragma unroll
            for (int kk = 0; kk < kTileTok / 16; ++kk) {
              const uint64_t da = tc::smem_desc_sw128(vt + kk * 16 * 128, kTileTok * 128, 1024);
              const uint64_t db = tc::smem_desc_sw128(ft + (kk / 4) * NF * 128 + (kk % 4) * 32, 16, 1024);
              tc::mma_ss(tmem + colC(cb), da, db, idesc_c, (t == 0 && kk == 0) ? 0u : 1u);
            }
            tc::commit(&bars[SB_KTEMPTY + ub]);
            tc::commit(&bars[SB_VEMPTY + vs]);
            if (t == x.n_tiles - 1) tc::commit(&bars[SB_CDONE + cb]);
          }
        }
        tc::commit(&bars[SB_DRAIN + 1]);
        tc::wait1(&bars[SB_DRAIN + 1], 0, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ feature groups (+ partial-state readout)
    const int w = warp < 8 ? 0 : 1;             // tile parity of this group
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;        // token of the tile / channel of C^T
    const int t128 = threadIdx.x - (w ? 256 : 128);
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    float2* stab = reinterpret_cast<float2*>(smem + S::kTab);
    if (w == 1) {
      // P_k (bf16, K-major, 128-byte swizzle) into shared memory for the U MMAs; with
      // head pairs the block-diagonal [P_k 0; 0 P_k] (slab hf holds rows hf r .. hf r + r - 1)
      if (PAIR) {
        for (int e = t128; e < 2 * NU * 8; e += 128) {
          const int hf = e / (NU * 8), n = (e / 8) % NU, c8 = e % 8;
          const uint4 v = (n / R == hf) ? __ldg(reinterpret_cast<const uint4*>(p_k + (n % R) * D) + c8)
                                        : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(smem + S::kPk + hf * NU * 128 + tc::sw128_offset(n, c8)) = v;
        }
      } else {
        for (int e = t128; e < R * (D / 8); e += 128) {
          const int n = e / (D / 8), c8 = e % (D / 8);
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(p_k + n * D) + c8);
          *reinterpret_cast<uint4*>(smem + S::kPk + (c8 / 8) * R * 128 + tc::sw128_offset(n, c8 % 8)) = v;
        }
      }
      if (S::kPool) {
        // block-membership tile: row 0 is 1 on tokens 0..63, row 1 on tokens 64..127, rows 2..15 zero
        for (int e = t128; e < 2 * 16 * 8; e += 128) {
          const int slab = e / (16 * 8), n = (e / 8) % 16, c = e % 8;
          const uint32_t one = (n == slab) ? 0x3f803f80u : 0u;  // two bf16 1.0
          *reinterpret_cast<uint4*>(smem + S::kInd + slab * 16 * 128 + tc::sw128_offset(n, c)) =
              make_uint4(one, one, one, one);
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[SB_PKREADY]);
    } else {
      // the RoPE table, shared by every token of the CTA
      if (tab_smem)
        for (int e = t128; e < tab_n; e += 128) stab[e] = __ldg(tab + e);
      tc::mbar_arrive(&bars[SB_TABREADY]);
    }
    const float2* rt = tab_smem ? stab : tab;
    bool ok = tc::wait_warp(&bars[SB_TABREADY], 0, abort_flag);
    int gi = 0, ii = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ii) {
      const Item x = item_of(P, n_chunks, n_sub, chunk_tok, it);
      for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
        if ((gi & 1) != w) continue;
        ok = tc::wait_warp(&bars[SB_UFULL + w], (gi >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        uint32_t ur[NU];
#pragma unroll
        for (int c = 0; c < NU / 16; ++c) tc::tmem_ld16p(tmem + lane_base + colU(w) + 16 * c, ur + 16 * c);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        tc::mbar_arrive(&bars[SB_UFREE + w]);
        const int hp = x.bh % HP;  // head (pair) of the item
        const int l = x.l0 + t * kTileTok + row;
        const bool valid = l < x.l1;  // rows past the piece (past L, or in the next causal chunk)
        const int lc = valid ? l : P.L - 1;
        const int gw = lc % P.grid_w;
        const int gh = (lc / P.grid_w) % P.grid_h;
        const int gt = lc / (P.grid_w * P.grid_h);
        const float2* tab_t = rt + gt * P.pairs_t;
        const float2* tab_h = rt + P.grid_t * P.pairs_t + gh * P.pairs_h - P.pairs_t;
        const float2* tab_w = rt + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + gw * P.pairs_w - P.pairs_t - P.pairs_h;
        uint32_t hd[NU], tl[NU];  // bf16 head / tail bit patterns of k~ (of both heads of a pair)
#pragma unroll
        for (int hh = 0; hh < NU / R; ++hh) {
          const bool vh = valid && (!PAIR || 2 * hp + hh < P.H);
#pragma unroll
          for (int mm = 0; mm < R / 2; ++mm) {
            const float xx = elu1_fast(__uint_as_float(ur[hh * R + 2 * mm]));
            const float yy = elu1_fast(__uint_as_float(ur[hh * R + 2 * mm + 1]));
            const float2* src = mm < P.pairs_t ? tab_t : (mm < P.pairs_t + P.pairs_h ? tab_h : tab_w);
            const float2 cs = src[mm];
            const float k0 = vh ? xx * cs.x - yy * cs.y : 0.f;
            const float k1 = vh ? xx * cs.y + yy * cs.x : 0.f;
            split_bits(k0, hd[hh * R + 2 * mm], tl[hh * R + 2 * mm]);
            split_bits(k1, hd[hh * R + 2 * mm + 1], tl[hh * R + 2 * mm + 1]);
          }
        }
        ok = tc::wait_warp(&bars[SB_KTEMPTY + w], ((gi >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        // features K-major: element (rank row, token `row`) of [2 token slabs][NF rows][128 B]:
        // per head of the item 2r rows, its head part in the first r, its tail in the next r
        unsigned char* ft = smem + S::kKt + w * S::kKtBytes + (row / 64) * NF * 128;
        const uint32_t chunk = (row % 64) / 8, within = (row % 8) * 2;
#pragma unroll
        for (int n = 0; n < NU; ++n) {
          const int base = (n / R) * 2 * R + n % R;
          *reinterpret_cast<uint16_t*>(ft + tc::sw128_offset(base, chunk) + within) = static_cast<uint16_t>(hd[n]);
          *reinterpret_cast<uint16_t*>(ft + tc::sw128_offset(base + R, chunk) + within) = static_cast<uint16_t>(tl[n]);
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bars[SB_KTFULL + w]);
        if (pool) {
          // block means of K for the tile's two blocks: thread = channel `row`
          ok = tc::wait_warp(&bars[SB_PFULL + w], (gi >> 1) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          uint32_t s0, s1;
          tc::tmem_ld2(tmem + lane_base + colP(w), s0, s1);
          tc::tmem_wait_ld();
          tc::fence_before_sync();
          tc::mbar_arrive(&bars[SB_PFREE + w]);
          const int b = x.bh / HP;
          const int h = PAIR ? 2 * hp + row / 64 : hp;  // channel row `row` belongs to head h
          const int ch = PAIR ? row % 64 : row;
          const int kb0 = (x.l0 + t * kTileTok) / 64;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kb = kb0 + e;
            if (kb >= P.n_kblk || h >= P.H) break;
            const int n_valid = min(64, P.L - kb * 64);
            float hdv, tlv;
            split_bf16(__uint_as_float(e ? s1 : s0) * (1.0f / static_cast<float>(n_valid)), hdv, tlv);
            uint16_t* dst = k_mean + ((static_cast<size_t>(b) * P.H + h) * P.n_kblk + kb) * 2 * D;
            const __nv_bfloat16 hb = __float2bfloat16_rn(hdv), tb = __float2bfloat16_rn(tlv);
            dst[ch] = *reinterpret_cast<const uint16_t*>(&hb);
            dst[D + ch] = *reinterpret_cast<const uint16_t*>(&tb);
          }
        }
      }
      if (!ok) break;
      if (w == 0) {
        // partial state of item ii: thread `row` holds channel row of C^T (head + tail parts);
        // with head pairs rows 64.. are the second head's, in the second half of the columns
        const int cb = ii & 1;
        ok = tc::wait_warp(&bars[SB_CDONE + cb], (ii >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const int hh = PAIR ? row / 64 : 0;  // the same for the whole warp
        uint32_t cr[2 * R];
#pragma unroll
        for (int c = 0; c < 2 * R / 16; ++c)
          tc::tmem_ld16p(tmem + lane_base + colC(cb) + hh * 2 * R + 16 * c, cr + 16 * c);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        tc::mbar_arrive(&bars[SB_CFREE + cb]);
        const int b = x.bh / HP, hp = x.bh % HP;
        const int h = PAIR ? 2 * hp + hh : hp;
        const int ch = PAIR ? row % 64 : row;
        if (h < P.H) {
          float* out = c_part + ((static_cast<size_t>(b) * P.H + h) * n_chunks + x.chunk) * R * D;
#pragma unroll
          for (int m = 0; m < R; ++m) out[m * D + ch] = __uint_as_float(cr[m]) + __uint_as_float(cr[R + m]);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) report_status(status, kStatusTimeout);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

bool make_map(CUtensorMap* map, const void* base, const Problem& P, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(P.d), static_cast<cuuint64_t>(P.H),
                              static_cast<cuuint64_t>(P.L), static_cast<cuuint64_t>(P.B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(P.d) * 2, static_cast<cuuint64_t>(P.H) * P.d * 2,
                                 static_cast<cuuint64_t>(P.L) * P.H * P.d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, bool PAIR>
cudaError_t run_state_tc(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k, uint16_t* k_mean,
                         const uint16_t* v, const uint16_t* p_k, float* c_part, unsigned* status,
                         cudaStream_t stream) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, P, kTileTok) || !make_map(&mv, v, P, kTileTok)) return cudaErrorInvalidValue;
  const int smem = StateSmem<R, PAIR>::kTotal + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(lowrank_state_tc_kernel<R, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = P.B * (PAIR ? (P.H + 1) / 2 : P.H) * lay.n_split;
  const int grid = n_items < sms ? n_items : sms;
  lowrank_state_tc_kernel<R, PAIR><<<grid, kThreads, smem, stream>>>(mk, mv, P, lay.n_split, lay.n_sub,
                                                                    lay.split_len, tab, p_k, c_part, k_mean, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// readout: O_lr = RMSNorm(q~^T C), tcgen05, d = 128, r <= 32
// ---------------------------------------------------------------------------
// Persistent: CTA c takes the contiguous run [c*I/G, (c+1)*I/G) of the items
// (batch, head, causal chunk, 128-token tile of the chunk), so C^T changes at
// most a few times per CTA; a tile that ends inside its chunk stores its rows
// directly instead of by TMA.
// Warps: 0 TMA (Q tiles into a 3-stage ring; C^T head and tail per head);
// 1 MMA issuer and TMEM owner: U = Q P_q^T (N = r) per tile, then, one tile
// behind, X = q~ (C_head + C_tail) as head*head + head*tail + tail*head (N = d);
// 4..7 features: q~ = R_r(p) phi(U) as a bf16 head (row bytes 0..63) and tail
// (row bytes 64..127) of one K-major 128-byte-swizzled row per token;
// 8..11 epilogue: o = X / sqrt(mean X^2 + eps) in bf16, out by TMA.
// U, q~ and X are double-buffered across tiles; all waits are bounded.

constexpr int kRdQStages = 3;

template <int R>
struct ReadSmem {
  static constexpr int kTileBytes = 2 * kTileTok * 128;  // one Q / O tile: 2 channel slabs x 128 rows x 128 B
  static constexpr int kSlab = 128 * 128;                // [128 rows][128 B]
  static constexpr int kQ = 0;                           // kRdQStages Q tiles
  static constexpr int kC = kQ + kRdQStages * kTileBytes;  // C^T head slab, tail slab ([d rows][64 ranks])
  static constexpr int kPq = kC + 2 * kSlab;             // P_q: 2 channel slabs x R rows x 128 B
  static constexpr int kQt = kPq + 2 * 32 * 128;         // 2 q~ buffers of one slab
  static constexpr int kOut = kQt + 2 * kSlab;           // output tile staging
  static constexpr int kTab = kOut + kTileBytes;
  static constexpr int kBars = kTab + kTabBytes;
  static constexpr int kTotal = kBars + 256;
};

enum {
  RB_QFULL = 0, RB_QEMPTY = RB_QFULL + kRdQStages, RB_CFULL = RB_QEMPTY + kRdQStages, RB_CEMPTY = RB_CFULL + 1,
  RB_PKREADY = RB_CEMPTY + 1, RB_UFULL = RB_PKREADY + 1, RB_UFREE = RB_UFULL + 2, RB_QTFULL = RB_UFREE + 2,
  RB_QTEMPTY = RB_QTFULL + 2, RB_XFULL = RB_QTEMPTY + 2, RB_XFREE = RB_XFULL + 2, RB_DRAIN = RB_XFREE + 2,
  RB_N = RB_DRAIN + 1
};

// Items (batch, head, causal chunk, tile of the chunk): tiles tile every chunk
// on its own (the whole sequence without a window), so a tile reads one C^T.
struct RdItem {
  int b, h, c, l0, rows;  // rows: of the tile's 128, those inside its chunk (and below L)
  bool head_start;        // a new (batch, head, chunk): its C^T is loaded
};
template <bool CAUSAL>
__device__ __forceinline__ RdItem rd_item(const Problem& P, int tpc, int it, int beg) {
  RdItem x;
  const int g = it / tpc, t = it % tpc;
  x.c = CAUSAL ? g % P.n_chunks : 0;
  const int bh = CAUSAL ? g / P.n_chunks : g;
  x.b = bh / P.H;
  x.h = bh % P.H;
  x.l0 = x.c * P.chunk_tokens + t * kTileTok;
  x.rows = min(kTileTok, min(P.L, chunk_end(P, x.c)) - x.l0);
  x.head_start = it == beg || t == 0;
  return x;
}

template <int R, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
lowrank_readout_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                          const __grid_constant__ CUtensorMap tm_ch, const __grid_constant__ CUtensorMap tm_cl,
                          Problem P, const float2* __restrict__ tab, const uint16_t* __restrict__ p_q,
                          uint16_t* __restrict__ o_lr, unsigned* status) {
  constexpr int D = 128;
  using S = ReadSmem<R>;
  constexpr uint32_t kCols = 512;  // U0, U1 at [0, 2r); X0 at [128, 256); X1 at [256, 384)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * RB_N);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * RB_N + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles = (P.chunk_tokens + kTileTok - 1) / kTileTok;  // per chunk
  const int n_items = P.B * P.H * P.n_chunks * n_tiles;
  const int beg = static_cast<int>(static_cast<long long>(blockIdx.x) * n_items / gridDim.x);
  const int end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * n_items / gridDim.x);
  const int tab_n = rope_table_entries(P);
  const bool tab_smem = tab_n * 8 <= kTabBytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRdQStages; ++s) {
      tc::mbar_init(&bars[RB_QFULL + s], 1);
      tc::mbar_init(&bars[RB_QEMPTY + s], 1);
    }
    tc::mbar_init(&bars[RB_CFULL], 1);
    tc::mbar_init(&bars[RB_CEMPTY], 1);
    tc::mbar_init(&bars[RB_PKREADY], 128);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[RB_UFULL + s], 1);
      tc::mbar_init(&bars[RB_UFREE + s], 128);
      tc::mbar_init(&bars[RB_QTFULL + s], 128);
      tc::mbar_init(&bars[RB_QTEMPTY + s], 1);
      tc::mbar_init(&bars[RB_XFULL + s], 1);
      tc::mbar_init(&bars[RB_XFREE + s], 128);
    }
    tc::mbar_init(&bars[RB_DRAIN], 1);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
    tc::tma_prefetch(&tm_o);
    tc::tma_prefetch(&tm_ch);
    tc::tma_prefetch(&tm_cl);
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto colU = [](int b) { return static_cast<uint32_t>(b * R); };
  auto colX = [](int b) { return static_cast<uint32_t>(128 + b * 128); };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      volatile int never = 0;
      bool ok = true;
      int gc = 0, gi = 0;  // C^T loads and Q tiles issued
      for (int it = beg; it < end && ok; ++it) {
        const RdItem x = rd_item<CAUSAL>(P, n_tiles, it, beg);
        const int st = gi % kRdQStages;
        ok = tc::wait1(&bars[RB_QEMPTY + st], ((gi / kRdQStages) & 1) ^ 1, abort_flag);
        if (!ok) break;
        unsigned char* dst = smem + S::kQ + st * S::kTileBytes;
        tc::mbar_arrive_expect_tx(&bars[RB_QFULL + st], S::kTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          tc::tma_load_4d(dst + hf * kTileTok * 128, &tm_q, &bars[RB_QFULL + st], 64 * hf, x.h, x.l0, x.b);
        ++gi;
        // C^T of a new head after that head's first Q tile: the X MMA that frees
        // the old C^T is issued behind the U MMA of this tile
        if (x.head_start) {
          if (gc > 0) ok = tc::wait1(&bars[RB_CEMPTY], (gc - 1) & 1, abort_flag);
          if (!ok) break;
          const int crow = ((x.b * P.H + x.h) * P.n_chunks + x.c) * D;
          tc::mbar_arrive_expect_tx(&bars[RB_CFULL], 2 * S::kSlab);
          tc::tma_load_2d(smem + S::kC, &tm_ch, &bars[RB_CFULL], 0, crow);
          tc::tma_load_2d(smem + S::kC + S::kSlab, &tm_cl, &bars[RB_CFULL], 0, crow);
          ++gc;
        }
      }
      // let the loads in flight land before the CTA can exit
      if (gc > 0) tc::wait1(&bars[RB_CFULL], (gc - 1) & 1, &never);
      for (int j = gi - kRdQStages < 0 ? 0 : gi - kRdQStages; j < gi; ++j)
        tc::wait1(&bars[RB_QFULL + j % kRdQStages], (j / kRdQStages) & 1, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      volatile int never = 0;
      constexpr uint32_t idesc_u = tc::idesc_bf16(128, R, false);
      constexpr uint32_t idesc_x = tc::idesc_bf16(128, D, false);
      bool ok = tc::wait1(&bars[RB_PKREADY], 0, abort_flag);
      if (ok) tc::fence_after_sync();
      int gcx = 0;  // C^T phases consumed by the X MMAs
      // X of the tile t (item beg + t): q~ and C^T in shared memory
      auto issue_x = [&](int t) -> bool {
        const int it = beg + t;
        const RdItem x = rd_item<CAUSAL>(P, n_tiles, it, beg);
        const bool head_end = it == end - 1 || (it + 1) % n_tiles == 0;
        const int qb = t & 1;
        bool good = true;
        if (x.head_start) good = tc::wait1(&bars[RB_CFULL], (gcx++) & 1, abort_flag);
        if (good) good = tc::wait1(&bars[RB_QTFULL + qb], (t >> 1) & 1, abort_flag);
        if (good && t >= 2) good = tc::wait1(&bars[RB_XFREE + qb], ((t >> 1) - 1) & 1, abort_flag);
        if (!good) return false;
        tc::fence_after_sync();
        const unsigned char* qt = smem + S::kQt + qb * S::kSlab;
        const unsigned char* ch = smem + S::kC;
        const unsigned char* cl = smem + S::kC + S::kSlab;
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t ah = tc::smem_desc_sw128(qt + 32 * kk, 16, 1024);
          const uint64_t at = tc::smem_desc_sw128(qt + 64 + 32 * kk, 16, 1024);
          const uint64_t bh = tc::smem_desc_sw128(ch + 32 * kk, 16, 1024);
          const uint64_t bl = tc::smem_desc_sw128(cl + 32 * kk, 16, 1024);
          tc::mma_ss(tmem + colX(qb), ah, bh, idesc_x, kk > 0 ? 1u : 0u);
          tc::mma_ss(tmem + colX(qb), ah, bl, idesc_x, 1u);
          tc::mma_ss(tmem + colX(qb), at, bh, idesc_x, 1u);
        }
        tc::commit(&bars[RB_XFULL + qb]);
        tc::commit(&bars[RB_QTEMPTY + qb]);
        if (head_end) tc::commit(&bars[RB_CEMPTY]);
        return true;
      };
      int gi = 0;
      for (int it = beg; it < end && ok; ++it, ++gi) {
        const int st = gi % kRdQStages, ub = gi & 1;
        ok = tc::wait1(&bars[RB_QFULL + st], (gi / kRdQStages) & 1, abort_flag);
        if (ok && gi >= 2) ok = tc::wait1(&bars[RB_UFREE + ub], ((gi >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const unsigned char* qtile = smem + S::kQ + st * S::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk / 4, c = kk % 4;
          const uint64_t da = tc::smem_desc_sw128(qtile + hf * kTileTok * 128 + c * 32, 16, 1024);
          const uint64_t db = tc::smem_desc_sw128(smem + S::kPq + hf * R * 128 + c * 32, 16, 1024);
          tc::mma_ss(tmem + colU(ub), da, db, idesc_u, kk > 0 ? 1u : 0u);
        }
        tc::commit(&bars[RB_UFULL + ub]);
        tc::commit(&bars[RB_QEMPTY + st]);
        if (gi >= 1) ok = issue_x(gi - 1);
      }
      if (ok && gi >= 1) issue_x(gi - 1);
      tc::commit(&bars[RB_DRAIN]);
      tc::wait1(&bars[RB_DRAIN], 0, &never);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ features
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const int t128 = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    float2* stab = reinterpret_cast<float2*>(smem + S::kTab);
    // P_q (bf16, K-major, 128-byte swizzle) for the U MMAs; the RoPE table
    for (int e = t128; e < R * (D / 8); e += 128) {
      const int n = e / (D / 8), c8 = e % (D / 8);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p_q + n * D) + c8);
      *reinterpret_cast<uint4*>(smem + S::kPq + (c8 / 8) * R * 128 + tc::sw128_offset(n, c8 % 8)) = v;
    }
    if (tab_smem)
      for (int e = t128; e < tab_n; e += 128) stab[e] = __ldg(tab + e);
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars[RB_PKREADY]);
    tc::named_barrier(1, 128);  // the table is complete before any row reads it
    const float2* rt = tab_smem ? stab : tab;
    bool ok = true;
    int gi = 0;
    for (int it = beg; it < end && ok; ++it, ++gi) {
      const RdItem x = rd_item<CAUSAL>(P, n_tiles, it, beg);
      const int ub = gi & 1;
      ok = tc::wait_warp(&bars[RB_UFULL + ub], (gi >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::fence_after_sync();
      uint32_t ur[R];
#pragma unroll
      for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(tmem + lane_base + colU(ub) + 16 * c, ur + 16 * c);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[RB_UFREE + ub]);
      const int l = x.l0 + row;
      const int lc = l < P.L ? l : P.L - 1;  // rows past L are computed but not stored
      const int gw = lc % P.grid_w;
      const int gh = (lc / P.grid_w) % P.grid_h;
      const int gt = lc / (P.grid_w * P.grid_h);
      const float2* tab_t = rt + gt * P.pairs_t;
      const float2* tab_h = rt + P.grid_t * P.pairs_t + gh * P.pairs_h - P.pairs_t;
      const float2* tab_w = rt + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + gw * P.pairs_w - P.pairs_t - P.pairs_h;
      uint32_t hd[R / 2], tl[R / 2];  // bf16 pairs (ranks 2mm, 2mm+1) of the head and the tail
#pragma unroll
      for (int mm = 0; mm < R / 2; ++mm) {
        const float xx = elu1_fast(__uint_as_float(ur[2 * mm]));
        const float yy = elu1_fast(__uint_as_float(ur[2 * mm + 1]));
        const float2* src = mm < P.pairs_t ? tab_t : (mm < P.pairs_t + P.pairs_h ? tab_h : tab_w);
        const float2 cs = src[mm];
        const float q0 = xx * cs.x - yy * cs.y;
        const float q1 = xx * cs.y + yy * cs.x;
        uint32_t h0, t0, h1, t1;
        split_bits(q0, h0, t0);
        split_bits(q1, h1, t1);
        hd[mm] = h0 | (h1 << 16);
        tl[mm] = t0 | (t1 << 16);
      }
      const int qb = gi & 1;
      ok = tc::wait_warp(&bars[RB_QTEMPTY + qb], ((gi >> 1) & 1) ^ 1, abort_flag);
      if (!ok) break;
      // row `row` of q~ (K-major, 128-byte swizzle): head ranks in chunks
      // 0..R/8-1, tail ranks in chunks 4..4+R/8-1
      unsigned char* qt = smem + S::kQt + qb * S::kSlab;
#pragma unroll
      for (int c = 0; c < R / 8; ++c) {
        *reinterpret_cast<uint4*>(qt + tc::sw128_offset(row, c)) =
            make_uint4(hd[4 * c], hd[4 * c + 1], hd[4 * c + 2], hd[4 * c + 3]);
        *reinterpret_cast<uint4*>(qt + tc::sw128_offset(row, 4 + c)) =
            make_uint4(tl[4 * c], tl[4 * c + 1], tl[4 * c + 2], tl[4 * c + 3]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[RB_QTFULL + qb]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const int t128 = threadIdx.x - 256;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    unsigned char* otile = smem + S::kOut;
    int gi = 0;
    for (int it = beg; it < end; ++it, ++gi) {
      const RdItem x = rd_item<CAUSAL>(P, n_tiles, it, beg);
      const int xb = gi & 1;
      const bool fail = !tc::wait_warp(&bars[RB_XFULL + xb], (gi >> 1) & 1, abort_flag) || *abort_flag;
      if (tc::named_barrier_or(2, 128, fail)) break;  // the four warps leave together
      tc::fence_after_sync();
      // pass 1: sum of squares of the row; pass 2 re-reads X, scales, packs
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + lane_base + colX(xb) + 32 * c, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ss += __uint_as_float(r[e]) * __uint_as_float(r[e]);
      }
      const float inv = rsqrtf(ss / D + P.rms_eps);
      // the previous tile's store must be done reading the staging tile; a tile that
      // ends inside its chunk stores its rows directly (a TMA box would overwrite
      // the next chunk's first rows)
      if (t128 == 0) tc::bulk_wait_group_read0();
      tc::named_barrier(2, 128);
      const bool direct = CAUSAL && x.rows < kTileTok;  // (rows past L alone are clipped by the TMA)
      if (!direct) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tc::tmem_ld32(tmem + lane_base + colX(xb) + 32 * c, r);
          tc::tmem_wait_ld();
          if (c == D / 32 - 1) {
            tc::fence_before_sync();
            tc::mbar_arrive(&bars[RB_XFREE + xb]);
          }
          // channels 32c .. 32c+31: half c/2 of the tile, chunks 4(c%2) .. 4(c%2)+3
          unsigned char* half = otile + (c / 2) * kTileTok * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t* v = r + 8 * k;
            const uint4 pk = make_uint4(
                pack_bf16(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                pack_bf16(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                pack_bf16(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                pack_bf16(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
            *reinterpret_cast<uint4*>(half + tc::sw128_offset(row, 4 * (c % 2) + k)) = pk;
          }
        }
      } else {
        // rows inside the chunk, straight to global memory
        uint16_t* orow = o_lr + ((static_cast<size_t>(x.b) * P.L + x.l0 + (row < x.rows ? row : 0)) * P.H + x.h) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tc::tmem_ld32(tmem + lane_base + colX(xb) + 32 * c, r);
          tc::tmem_wait_ld();
          if (c == D / 32 - 1) {
            tc::fence_before_sync();
            tc::mbar_arrive(&bars[RB_XFREE + xb]);
          }
          if (row < x.rows) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t* v = r + 8 * k;
              *reinterpret_cast<uint4*>(orow + 32 * c + 8 * k) = make_uint4(
                  pack_bf16(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                  pack_bf16(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                  pack_bf16(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                  pack_bf16(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
            }
          }
        }
      }
      tc::fence_proxy_async_smem();
      tc::named_barrier(2, 128);
      if (t128 == 0 && !direct) {
        for (int hf = 0; hf < 2; ++hf) tc::tma_store_4d(&tm_o, otile + hf * kTileTok * 128, 64 * hf, x.h, x.l0, x.b);
        tc::bulk_commit_group();
      }
    }
    if (t128 == 0) tc::bulk_wait_group0();
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) report_status(status, kStatusTimeout);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
}

// C^T head or tail, [B*H*n_chunks*d rows, r] bf16, as 128-byte rows of 64 ranks
// (ranks past r read as zero) of d rows: one box per (batch, head, causal chunk).
bool make_ct_map(CUtensorMap* map, const void* base, const Problem& P) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(P.rank),
                              static_cast<cuuint64_t>(P.B) * P.H * P.n_chunks * P.d};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(P.rank) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(P.d)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R>
cudaError_t run_readout_tc(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                           const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr, unsigned* status,
                           cudaStream_t stream) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap mq, mo, mch, mcl;
  if (!make_map(&mq, q, P, kTileTok) || !make_map(&mo, o_lr, P, kTileTok) || !make_ct_map(&mch, ct_hi, P) ||
      !make_ct_map(&mcl, ct_lo, P))
    return cudaErrorInvalidValue;
  const int smem = ReadSmem<R>::kTotal + 1024;
  auto kern = P.causal ? lowrank_readout_tc_kernel<R, true> : lowrank_readout_tc_kernel<R, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long n_items =
      static_cast<long long>(P.B) * P.H * P.n_chunks * ((P.chunk_tokens + kTileTok - 1) / kTileTok);
  const int grid = static_cast<int>(n_items < sms ? n_items : sms);
  kern<<<grid, kThreads, smem, stream>>>(mq, mo, mch, mcl, P, tab, p_q, o_lr, status);
  return cudaGetLastError();
}

}  // namespace

// Tokens per work item: 2048, halved (down to 256) while the problem would
// give fewer items than kItemsWanted, so short sequences still spread over
// every SM. A multiple of the 128-token tile and of the 64-token key block.
int lowrank_state_tc_chunk(const Problem& P) {
  const long long bh = static_cast<long long>(P.B) * P.H;
  int chunk = kChunkTok;
  while (chunk > kChunkMin && bh * ((P.L + chunk - 1) / chunk) < kItemsWanted) chunk /= 2;
  return chunk;
}

// d = 64 runs with two heads per tile, for r <= 32 (room in TMEM and shared memory).
bool lowrank_state_tc_supported(const Problem& P) { return P.d == 128 || (P.d == 64 && P.rank <= 32); }

// The key block means come out of the state pass only without a causal window
// (the selector pools the chunks' edge blocks itself).
bool lowrank_state_tc_pools_k(const Problem& P) { return lowrank_state_tc_supported(P) && P.rank <= 32 && !P.causal; }

cudaError_t launch_lowrank_state_tc(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                                    uint16_t* k_mean,
                                    const uint16_t* v, const uint16_t* p_k, float* c_part, unsigned* status,
                                    cudaStream_t stream) {
  if (P.d == 64) {
    if (P.rank == 16) return run_state_tc<16, true>(P, lay, tab, k, k_mean, v, p_k, c_part, status, stream);
    if (P.rank == 32) return run_state_tc<32, true>(P, lay, tab, k, k_mean, v, p_k, c_part, status, stream);
    return cudaErrorInvalidValue;
  }
  if (P.rank == 16) return run_state_tc<16, false>(P, lay, tab, k, k_mean, v, p_k, c_part, status, stream);
  if (P.rank == 32) return run_state_tc<32, false>(P, lay, tab, k, k_mean, v, p_k, c_part, status, stream);
  if (P.rank == 64) return run_state_tc<64, false>(P, lay, tab, k, nullptr, v, p_k, c_part, status, stream);
  return cudaErrorInvalidValue;
}

bool lowrank_readout_tc_supported(const Problem& P) { return P.d == 128 && (P.rank == 16 || P.rank == 32); }

cudaError_t launch_lowrank_readout_tc(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                                      const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr,
                                      unsigned* status, cudaStream_t stream) {
  if (P.rank == 16) return run_readout_tc<16>(P, tab, q, p_q, ct_hi, ct_lo, o_lr, status, stream);
  if (P.rank == 32) return run_readout_tc<32>(P, tab, q, p_q, ct_hi, ct_lo, o_lr, status, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sda
