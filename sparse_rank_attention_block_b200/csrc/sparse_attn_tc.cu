// Block-sparse attention A_M on the 5th-generation tensor cores (tcgen05),
// optionally with the low-rank readout and the gate fused into its epilogue
// (SparkDiffusion summary, robotworld.top, section 2.1: softmax(Q K^T /
// sqrt(d)) V restricted to the kept key blocks; O_lr = RMSNorm(q~^T C) with
// q~ = R_r(p) phi(P_q q); O = O_s + g r O_lr).
//
// One CTA per (batch, head, 128-row query block). The kept key blocks are
// taken two at a time (a 128-key step j); even and odd steps form two
// independent pipelines w = j % 2, each with its own S buffer (TMEM), P
// buffer (shared memory), K and V stages, softmax state (m, l) and output
// accumulator O_w (TMEM), merged once at the end.
//
// A single thread issuing tcgen05.mma keeps about one instruction in flight,
// so a 128x128x16 MMA chain from one thread runs at roughly half the tensor
// pipe's rate; four issuing warps keep it busy. Warps:
//   0  QK issuer of the even steps (S_j = Q K_j^T into S_0), TMA of Q and of
//      the even K tiles; fused form: X = q~ C at the end;
//   1  QK issuer of the odd steps, TMA of their K tiles; TMEM owner; fused
//      form: U = Q P_q^T at the start;
//   2  PV issuer of the even steps (O_0 += P_j V_j, P and V from shared
//      memory), TMA of their V tiles;
//   3  the same for the odd steps;
//   4..7  softmax of the even steps, then the epilogue;
//   8..11 softmax of the odd steps; fused form: the low-rank features q~ of
//         the tile at the start and the C^T tiles at the end.
// The softmax reads S_j out of TMEM and releases the S buffer at once (so
// QK_{j+2} overlaps the rest of the step), computes P_j = 2^(s*scale - m)
// in fp32 (log2 units, scale log2(e)/sqrt(d)), writes it as bf16 into its P
// buffer and hands it to the PV issuer. m moves, and O_w is rescaled in
// TMEM, only when the row max grows by more than 2^8, which is exact because
// numerator and denominator share m. A fixed share (kEmuPairs) of the
// exponentials on full blocks can run on the FMA pipe (ex2_fma2) instead of
// the MUFU unit.
//
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d),
// O_1 [384,384+d). Fused form: U lands in O_1 before the first odd PV; at
// the end q~ (bf16 head | tail) sits in S_1 and X = q~ (C_head + C_tail) in S_0.
// Shared memory: Q tile, K stage per pipeline, V stage per pipeline, P buffer
// per pipeline (P_1 also carries P_q at the start and C^T at the end, P_0 the
// output tile for the TMA store), barriers.
//
// Epilogue: O_s = (e0 O_0 + e1 O_1) / l with the merged softmax state; the
// fused form adds g r X / sqrt(mean X^2 + eps), r the RMS of the fp32 O_s row.
// Every wait is bounded (2 s; the waits on pipeline progress take the limit
// set by sda_set_attention_wait_limit); a CTA that gives up reports through
// the status word, drains its TMA loads and MMAs, frees TMEM and exits.

#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <type_traits>

#include <mutex>

#include "common.cuh"
#include "ex2_fma.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kThreads = 384;   // 12 warps, 3 per SM sub-partition
constexpr int kBQ = 128;
constexpr int kBK = 64;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
constexpr int kWarpEven = 4;    // first warp of the even-step softmax group
constexpr int kWarpOdd = 8;     // first warp of the odd-step softmax group
// Exponentials per 16 column pairs of a full block that run on the FMA pipe
// (ex2_fma2) instead of MUFU. Measured on the 720P, 480P and 8k-token layers
// (0, 2, 4, 6, 8 of 16, two alternating runs each): 0 is fastest (by ~2 % at
// full clock against 4): the emulation's extra instructions cost more issue
// slots than the MUFU time they save.
constexpr int kEmuPairs = 0;
// Register split: launched at kRegsLaunch per thread; the issuing warpgroup
// drops to kRegsLow, the two softmax groups rise to kRegsHigh.
constexpr int kRegsLaunch = 168, kRegsLow = 56, kRegsHigh = 224;
static_assert(kRegsLow * 128 + kRegsHigh * 256 <= kRegsLaunch * kThreads, "register split exceeds the launch");

template <int D, int R, bool FUSED>
struct Smem {
  static constexpr int kHalves = D / 64;                    // 64-element (128-byte) column slabs
  static constexpr int kQBytes = kHalves * kBQ * 128;        // [half][128 rows][128 B]
  static constexpr int kKVBytes = kHalves * 2 * kBK * 128;   // [half][128 keys][128 B]
  static constexpr int kPBytes = 2 * kBQ * 128;              // P: [key half][128 rows][128 B] bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;                    // one stage per pipeline
  static constexpr int kV = kK + 2 * kKVBytes;               // one stage per pipeline
  static constexpr int kP = kV + 2 * kKVBytes;               // one buffer per pipeline
  static constexpr int kBars = kP + 2 * kPBytes;
  static constexpr int kMerge = kBars + 256;                 // (m, l) of the odd pipeline, per row
  static constexpr int kTotal = kMerge + 2 * kBQ * 4;
  // fused form: P_q [half][r rows][128 B] (and the RoPE table) in P_1 at the
  // start; C^T head and tail [d rows][128 B] each in the odd K stage at the end
  static constexpr int kCtBytes = D * 128;
  static_assert(R * D * 2 <= 16384, "P_q must fit in front of the RoPE table");
  static_assert(2 * kCtBytes <= kKVBytes, "C^T tiles must fit in a K stage");
  static_assert(kHalves * kBQ * 128 <= kPBytes, "output tile must fit in a P buffer");
};

// barrier slots (two per pipeline where indexed by w)
enum {
  B_QFULL = 0, B_KFULL = 1, B_VFULL = 3, B_SFULL = 5, B_SFREE = 7, B_PFULL = 9, B_ODONE = 11,
  B_PQREADY = 13, B_UFULL = 14, B_QTREADY = 15, B_XFULL = 16, B_CTFULL = 17, B_DRAIN = 18,
  N_BARS = 22  // drain: one per issuer
};

struct FusedArgs {
  const uint16_t* p_q;     // [r, d] bf16
  const uint16_t* ct_hi;   // [B, H, d, r] bf16: C^T head
  const uint16_t* ct_lo;   // [B, H, d, r] bf16: C^T tail (C^T - head)
  const float2* rope_tab;  // cos/sin table (see common.cuh)
  const float* gate;       // [B, L] or [B, L, H]
  int tab_entries;         // table entries (float2); staged in shared memory when <= kTabMax
  float* lse;              // plain form, optional: per row (b, l, h) log2-sum-exp2 of the scaled scores
};

// The RoPE table is staged in P_1 behind P_q when it fits.
constexpr int kTabOffset = 16384, kTabMax = 16384 / 8;

// Feature helpers of the fused epilogue, kept off the quarter-rate conversion
// pipe: phi(u) = elu(u) + 1 with the fast exponential, and x split into a
// bf16 head (rounded half up, high 16 bits) and the fp32 remainder.
__device__ __forceinline__ float elu1_fast(float u) { return u > 0.f ? u + 1.f : __expf(u); }
__device__ __forceinline__ void split_bf16_int(float x, uint32_t& head_bits, float& tail) {
  head_bits = (__float_as_uint(x) + 0x8000u) & 0xffff0000u;
  tail = x - __uint_as_float(head_bits);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a [rows][128 B]
// tile with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw(uint32_t row, uint32_t chunk) { return tc::sw128_offset(row, chunk); }

template <int D, int R, bool FUSED, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_chi, const __grid_constant__ CUtensorMap tm_clo,
                      Problem P, const int32_t* __restrict__ block_idx, FusedArgs fa, unsigned* status,
                      uint64_t wait_ns) {
  using S = Smem<D, R, FUSED>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * N_BARS + 4);
  int* bad_flag = reinterpret_cast<int*>(smem + S::kBars + 8 * N_BARS + 8);
  float* merge_m = reinterpret_cast<float*>(smem + S::kMerge);
  float* merge_l = merge_m + kBQ;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // The CTA's 128-row tile: one 128-row query block, or two adjacent 64-row
  // query blocks a, a1 of the same causal chunk (a alone at a chunk's end,
  // the tile's second half then past the chunk: computed, never stored).
  constexpr bool pair = PAIR;  // P.block_q == 64
  const int tiles = pair ? P.n_chunks * ((P.nq_chunk + 1) / 2) : P.n_qblk;  // tiles per (batch, head)
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % P.H;
  const int b = blockIdx.x / (tiles * P.H);
  int a = tile, a1 = -1;
  if (pair) {
    const int per_chunk = (P.nq_chunk + 1) / 2, c = tile / per_chunk, m2 = 2 * (tile % per_chunk);
    a = c * P.nq_chunk + m2;
    if (m2 + 1 < P.nq_chunk) a1 = a + 1;
  }
  // Causal window: the tile lies in chunk cq and sees the keys below hi; a
  // query block keeps `keep` of its n_cand candidate blocks (the first entries
  // of its row). Without a window: cq = 0, hi = L, n_cand = N_kblk, keep = k.
  const int cq = qblk_chunk(P, a);
  const int hi = chunk_end(P, cq);
  const int n_cand = chunk_cands(P, cq);
  const int keep = keep_of(P, n_cand);
  const int q_row = (a - cq * P.nq_chunk) * P.block_q;  // Q/O map coordinates: row in the chunk, (batch, chunk) slab
  const int q_slab = b * P.n_chunks + cq;
  const int32_t* idx = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * P.keep;
  const int32_t* idx1 =
      (PAIR && a1 >= 0) ? block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a1) * P.keep : nullptr;
  int* n_entries_smem = reinterpret_cast<int*>(smem + S::kBars + 8 * N_BARS + 12);

  // A pair's key-block list is the ascending merge of its two map rows (entries
  // outside [0, n_cand) skipped and reported), each entry with the halves of
  // the tile that kept it (bit 0: rows 0-63, bit 1: rows 64-127). Every role
  // walks it with a cursor of its own, in step order.
  struct Cursor {
    int i0, i1, pos;
  };
  auto next_merged = [&](Cursor& c, int& blk, int& bits) {
    for (;;) {
      const int v0 = c.i0 < keep ? __ldg(idx + c.i0) : INT_MAX;
      const int v1 = (idx1 != nullptr && c.i1 < keep) ? __ldg(idx1 + c.i1) : INT_MAX;
      if (v0 != INT_MAX && (v0 < 0 || v0 >= n_cand)) {
        *bad_flag = 1;
        ++c.i0;
        continue;
      }
      if (v1 != INT_MAX && (v1 < 0 || v1 >= n_cand)) {
        *bad_flag = 1;
        ++c.i1;
        continue;
      }
      if (v0 == INT_MAX && v1 == INT_MAX) {
        blk = -2;
        bits = 0;
      } else if (v0 <= v1) {
        blk = v0;
        bits = v0 == v1 ? 3 : 1;
        ++c.i0;
        if (v0 == v1) ++c.i1;
      } else {
        blk = v1;
        bits = 2;
        ++c.i1;
      }
      return;
    }
  };

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars[B_QFULL], 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[B_KFULL + s], 1);
      tc::mbar_init(&bars[B_VFULL + s], 1);
      tc::mbar_init(&bars[B_SFULL + s], 1);
      tc::mbar_init(&bars[B_SFREE + s], 128);
      tc::mbar_init(&bars[B_PFULL + s], 128);
      tc::mbar_init(&bars[B_ODONE + s], 1);
      tc::mbar_init(&bars[B_DRAIN + s], 1);
      tc::mbar_init(&bars[B_DRAIN + 2 + s], 1);
    }
    tc::mbar_init(&bars[B_PQREADY], 128);
    tc::mbar_init(&bars[B_UFULL], 1);
    tc::mbar_init(&bars[B_QTREADY], 128);
    tc::mbar_init(&bars[B_XFULL], 1);
    tc::mbar_init(&bars[B_CTFULL], 1);
    // A CTA of this launch (or an unread earlier one) gave up a wait: the
    // outputs are undefined until the status is read, so do no more work.
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    *bad_flag = 0;
    if constexpr (PAIR) {  // length of the merged list
      Cursor c{0, 0, 0};
      int blk, bits, n_ent = 0;
      for (next_merged(c, blk, bits); blk >= 0; next_merged(c, blk, bits)) ++n_ent;
      *n_entries_smem = n_ent;
    }
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
    tc::tma_prefetch(&tm_o);
    if constexpr (FUSED) {
      tc::tma_prefetch(&tm_chi);
      tc::tma_prefetch(&tm_clo);
    }
  }
  __syncthreads();
  if (*abort_flag) return;  // uniform: every thread reads the same shared flag
  const int n_steps = ((PAIR ? *n_entries_smem : keep) + 1) / 2;  // two key blocks per step
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Key blocks of step j (fetched a step ahead of use, steps in increasing
  // order per cursor) and the halves that kept them, then checked: -1 marks
  // an invalid block, -2 a missing one (odd list length).
  auto fetch_blocks = [&](Cursor& c, int j, int& r0, int& r1, int& m0, int& m1) {
    if (!pair) {
      r0 = __ldg(idx + 2 * j);
      r1 = (2 * j + 1 < keep) ? __ldg(idx + 2 * j + 1) : -2;
      m0 = m1 = 3;
      return;
    }
    int blk, bits;
    for (; c.pos < 2 * j; ++c.pos) next_merged(c, blk, bits);
    next_merged(c, r0, m0);
    next_merged(c, r1, m1);
    c.pos += 2;
  };
  auto check_blocks = [&](int r0, int r1, int& b0, int& b1) {
    b0 = (r0 < 0 || r0 >= n_cand) ? -1 : r0;
    b1 = (r1 == -2) ? -2 : ((r1 < 0 || r1 >= n_cand) ? -1 : r1);
  };
  // TMA of the two key blocks of a step (K or V) into one stage; a missing or
  // invalid second block reloads the first one (its keys are masked)
  auto load_kv = [&](const CUtensorMap* map, unsigned char* dst, uint64_t* bar, int r0, int r1) {
    constexpr uint32_t kHalfBytes = kBK * 128;  // one 64-key x 64-element box
    int b0, b1;
    check_blocks(r0, r1, b0, b1);
    if (b0 == -1 || b1 == -1) *bad_flag = 1;
    const int lb0 = b0 >= 0 ? b0 : 0;
    const int lb1 = b1 >= 0 ? b1 : lb0;
    tc::mbar_arrive_expect_tx(bar, S::kKVBytes);
    for (int hf = 0; hf < S::kHalves; ++hf) {
      tc::tma_load_4d(dst + hf * 2 * kHalfBytes, map, bar, 64 * hf, h, lb0 * kBK, b);
      tc::tma_load_4d(dst + hf * 2 * kHalfBytes + kHalfBytes, map, bar, 64 * hf, h, lb1 * kBK, b);
    }
  };

  // Registers move from the issuing warpgroup to the two softmax groups; the
  // host checks that the launch holds enough for the split.
  if (warp < kWarpEven) {
    tc::setmaxnreg_dec<kRegsLow>();
    if (lane == 0) {
      const int w = warp & 1;  // pipeline
      volatile int never = 0;
      if (warp < 2) {
        // ---------------------------------------------------- QK issuer of pipeline w
        constexpr uint32_t idesc_qk = tc::idesc_bf16(128, 128, false);
        unsigned char* kst = smem + S::kK + w * S::kKVBytes;
        bool ok = true;
        bool q_pending = false;
        int k_pending = -1;  // group step of a K load issued but not yet waited for
        if (w == 0) {
          tc::mbar_arrive_expect_tx(&bars[B_QFULL], S::kQBytes);
          for (int hf = 0; hf < S::kHalves; ++hf)
            tc::tma_load_4d(smem + S::kQ + hf * kBQ * 128, &tm_q, &bars[B_QFULL], 64 * hf, h, q_row, q_slab);
          q_pending = true;
        }
        int nr0 = 0, nr1 = 0, nm0, nm1;  // indices of the next K tile of this pipeline
        Cursor cur{0, 0, 0};
        if (w < n_steps) {
          fetch_blocks(cur, w, nr0, nr1, nm0, nm1);
          load_kv(&tm_k, kst, &bars[B_KFULL + w], nr0, nr1);
          k_pending = 0;
          if (w + 2 < n_steps) fetch_blocks(cur, w + 2, nr0, nr1, nm0, nm1);
        }
        ok = tc::wait1(&bars[B_QFULL], 0, abort_flag, wait_ns);
        if (ok) q_pending = false;
        if constexpr (FUSED) {
          if (ok && w == 1) {
            // U = Q P_q^T into the O_1 columns (free until the first odd PV)
            ok = tc::wait1(&bars[B_PQREADY], 0, abort_flag, wait_ns);
            if (ok) {
              tc::fence_after_sync();
              constexpr uint32_t idesc_u = tc::idesc_bf16(128, R, false);
              const unsigned char* pq = smem + S::kP + S::kPBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const int hf = kk / 4, c = kk % 4;
                const uint64_t da = tc::smem_desc_sw128(smem + S::kQ + hf * kBQ * 128 + c * 32, 16, 1024);
                const uint64_t db = tc::smem_desc_sw128(pq + hf * R * 128 + c * 32, 16, 1024);
                tc::mma_ss(tmem + kColO1, da, db, idesc_u, kk > 0 ? 1u : 0u);
              }
              tc::commit(&bars[B_UFULL]);
            }
          }
        }
        int i = 0;
        for (int j = w; j < n_steps && ok; j += 2, ++i) {
          // S_w is free once the softmax has read S of the previous group step
          if (i > 0) ok = tc::wait1(&bars[B_SFREE + w], (i - 1) & 1, abort_flag, wait_ns);
          if (ok) ok = tc::wait1(&bars[B_KFULL + w], i & 1, abort_flag, wait_ns);
          if (!ok) break;
          k_pending = -1;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hf = kk / 4, c = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(smem + S::kQ + hf * kBQ * 128 + c * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(kst + hf * 2 * kBK * 128 + c * 32, 16, 1024);
            tc::mma_ss(tmem + (w ? kColS1 : kColS0), da, db, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[B_SFULL + w]);
          if (j + 2 < n_steps) {
            // the K stage is free once QK_j has completed
            ok = tc::wait1(&bars[B_SFULL + w], i & 1, abort_flag, wait_ns);
            if (!ok) break;
            load_kv(&tm_k, kst, &bars[B_KFULL + w], nr0, nr1);
            k_pending = i + 1;
            if (j + 4 < n_steps) fetch_blocks(cur, j + 4, nr0, nr1, nm0, nm1);
          }
        }
        bool ct_pending = false;
        if constexpr (FUSED) {
          if (ok && w == 1) {
            // C^T head / tail into the odd K stage once its last QK has completed
            const int n_w = n_steps / 2;
            if (n_w > 0) ok = tc::wait1(&bars[B_SFULL + 1], (n_w - 1) & 1, abort_flag, wait_ns);
            if (ok) {
              tc::mbar_arrive_expect_tx(&bars[B_CTFULL], 2 * S::kCtBytes);
              const int ct_row = static_cast<int>(((static_cast<size_t>(b) * P.H + h) * P.n_chunks + cq) * D);
              tc::tma_load_2d(kst, &tm_chi, &bars[B_CTFULL], 0, ct_row);
              tc::tma_load_2d(kst + S::kCtBytes, &tm_clo, &bars[B_CTFULL], 0, ct_row);
              ct_pending = true;
            }
          }
        }
        if constexpr (FUSED) {
          if (ok && w == 0) {
            // X = q~ (C_head + C_tail) into S_0 once the even softmax has read
            // its last S and the odd group has staged q~ and C^T
            const int n_w = (n_steps + 1) / 2;
            if (n_w > 0) ok = tc::wait1(&bars[B_SFREE], (n_w - 1) & 1, abort_flag, wait_ns);
            if (ok) ok = tc::wait1(&bars[B_QTREADY], 0, abort_flag, wait_ns);
            if (ok) ok = tc::wait1(&bars[B_CTFULL], 0, abort_flag, wait_ns);
            if (ok) {
              tc::fence_after_sync();
              constexpr uint32_t idesc_x = tc::idesc_bf16(128, D, false);
              const unsigned char* chi = smem + S::kK + S::kKVBytes;
              const unsigned char* clo = chi + S::kCtBytes;
              int n_mma = 0;
#pragma unroll
              for (int kk = 0; kk < R / 16; ++kk) {
                const uint64_t dh = tc::smem_desc_sw128(chi + kk * 32, 16, 1024);
                const uint64_t dl = tc::smem_desc_sw128(clo + kk * 32, 16, 1024);
                const uint32_t qh = tmem + kColS1 + kk * 8, ql = tmem + kColS1 + R / 2 + kk * 8;
                tc::mma_ts(tmem + kColS0, qh, dh, idesc_x, n_mma++ > 0 ? 1u : 0u);
                tc::mma_ts(tmem + kColS0, qh, dl, idesc_x, 1u);
                tc::mma_ts(tmem + kColS0, ql, dh, idesc_x, 1u);
              }
              tc::commit(&bars[B_XFULL]);
            }
          }
        }
        // drain: loads still in flight, then every MMA this thread issued
        if (q_pending) tc::wait1(&bars[B_QFULL], 0, &never);
        if (k_pending >= 0) tc::wait1(&bars[B_KFULL + w], k_pending & 1, &never);
        if (ct_pending) tc::wait1(&bars[B_CTFULL], 0, &never);
        tc::commit(&bars[B_DRAIN + warp]);
        tc::wait1(&bars[B_DRAIN + warp], 0, &never);
      } else {
        // ---------------------------------------------------- PV issuer of pipeline w
        constexpr uint32_t idesc_pv = tc::idesc_bf16(128, D, true);  // A = P K-major, B = V MN-major
        unsigned char* vst = smem + S::kV + w * S::kKVBytes;
        const unsigned char* pbuf = smem + S::kP + w * S::kPBytes;
        bool ok = true;
        int v_pending = -1;
        int nr0 = 0, nr1 = 0, nm0, nm1;  // indices of the next V tile of this pipeline
        Cursor cur{0, 0, 0};
        if (w < n_steps) {
          fetch_blocks(cur, w, nr0, nr1, nm0, nm1);
          load_kv(&tm_v, vst, &bars[B_VFULL + w], nr0, nr1);
          v_pending = 0;
          if (w + 2 < n_steps) fetch_blocks(cur, w + 2, nr0, nr1, nm0, nm1);
        }
        int i = 0;
        for (int j = w; j < n_steps && ok; j += 2, ++i) {
          ok = tc::wait1(&bars[B_PFULL + w], i & 1, abort_flag, wait_ns);
          if (ok) ok = tc::wait1(&bars[B_VFULL + w], i & 1, abort_flag, wait_ns);
          if (!ok) break;
          v_pending = -1;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 2 * kBK / 16; ++kk) {
            // 16 keys per MMA: A = P columns kk*16.. (key half kk/4), B = V rows kk*16..
            const uint64_t da = tc::smem_desc_sw128(pbuf + (kk / 4) * kBQ * 128 + (kk % 4) * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(vst + kk * 16 * 128, 2 * kBK * 128, 1024);
            tc::mma_ss(tmem + (w ? kColO1 : kColO0), da, db, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(&bars[B_ODONE + w]);
          if (j + 2 < n_steps) {
            // the V stage is free once PV_j has completed
            ok = tc::wait1(&bars[B_ODONE + w], i & 1, abort_flag, wait_ns);
            if (!ok) break;
            load_kv(&tm_v, vst, &bars[B_VFULL + w], nr0, nr1);
            v_pending = i + 1;
            if (j + 4 < n_steps) fetch_blocks(cur, j + 4, nr0, nr1, nm0, nm1);
          }
        }
        if (v_pending >= 0) tc::wait1(&bars[B_VFULL + w], v_pending & 1, &never);
        tc::commit(&bars[B_DRAIN + warp]);
        tc::wait1(&bars[B_DRAIN + warp], 0, &never);
      }
    }
  } else {
    tc::setmaxnreg_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax groups (+ epilogue)
    const int w = warp < kWarpOdd ? 0 : 1;        // pipeline: 0 even steps (and the epilogue), 1 odd steps
    const int quarter = warp & 3;                 // TMEM lanes [32*quarter, +32)
    const int row = 32 * quarter + lane;          // query row of the tile
    const int t128 = threadIdx.x - (w ? 32 * kWarpOdd : 32 * kWarpEven);  // 0..127 within the group
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    const uint32_t col_s = w ? kColS1 : kColS0;
    const uint32_t col_o = w ? kColO1 : kColO0;
    unsigned char* pbuf = smem + S::kP + w * S::kPBytes;
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const int tok = qblk_start(P, a) + row;
    const int tokc = tok < hi ? tok : hi - 1;  // rows past the chunk are computed, never stored
    bool ok = true;

    // fused form, odd group: stage P_q in P_1, then the features of this row
    // q~ = R_r(p) phi(U) from U = Q P_q^T, kept as bf16 head | tail pairs
    uint32_t qt[FUSED ? R : 1];
    if constexpr (FUSED) {
      if (w == 1) {
        for (int e = t128; e < R * (D / 8); e += 128) {
          const int n = e / (D / 8), c8 = e % (D / 8);  // row n, 16-byte chunk c8 (8 channels)
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(fa.p_q + n * D) + c8);
          *reinterpret_cast<uint4*>(pbuf + (c8 / 8) * R * 128 + sw(n, c8 % 8)) = v;
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bars[B_PQREADY]);
        // RoPE table into P_1 behind P_q (shared by every row of the tile)
        const bool tab_smem = fa.tab_entries <= kTabMax;
        float2* stab = reinterpret_cast<float2*>(pbuf + kTabOffset);
        if (tab_smem) {
          for (int e = t128; e < fa.tab_entries; e += 128) stab[e] = __ldg(fa.rope_tab + e);
          tc::named_barrier(2, 128);
        }
        const float2* tab = tab_smem ? stab : fa.rope_tab;
        ok = tc::wait_warp(&bars[B_UFULL], 0, abort_flag, wait_ns);
        if (ok) {
          tc::fence_after_sync();
          uint32_t ur[R];
#pragma unroll
          for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(tmem + lane_base + kColO1 + 16 * c, ur + 16 * c);
          tc::tmem_wait_ld();
          const int gw = tokc % P.grid_w;
          const int gh = (tokc / P.grid_w) % P.grid_h;
          const int gt = tokc / (P.grid_w * P.grid_h);
          // table rows of this token per axis, indexed by the global pair number
          const float2* tab_t = tab + gt * P.pairs_t;
          const float2* tab_h = tab + P.grid_t * P.pairs_t + gh * P.pairs_h - P.pairs_t;
          const float2* tab_w = tab + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + gw * P.pairs_w - P.pairs_t - P.pairs_h;
          float2 cs[R / 2];
#pragma unroll
          for (int mm = 0; mm < R / 2; ++mm) {
            const float2* src = mm < P.pairs_t ? tab_t : (mm < P.pairs_t + P.pairs_h ? tab_h : tab_w);
            cs[mm] = src[mm];
          }
#pragma unroll
          for (int mm = 0; mm < R / 2; ++mm) {
            const float x = elu1_fast(__uint_as_float(ur[2 * mm]));
            const float y = elu1_fast(__uint_as_float(ur[2 * mm + 1]));
            const float2 cs2 = cs[mm];
            const float k0 = x * cs2.x - y * cs2.y, k1 = x * cs2.y + y * cs2.x;
            uint32_t h0, h1;
            float t0, t1;
            split_bf16_int(k0, h0, t0);
            split_bf16_int(k1, h1, t1);
            qt[mm] = __byte_perm(h0, h1, 0x7632);
            qt[R / 2 + mm] = __byte_perm(__float_as_uint(t0) + 0x8000u, __float_as_uint(t1) + 0x8000u, 0x7632);
          }
        }
        // every row has read the table before any P_1 overwrites it
        if (tab_smem) tc::named_barrier(2, 128);
      }
    }

    float m = -INFINITY;  // reference max (log2 units)
    float l = 0.f;
    int i = 0;            // step number within the pipeline
    int nr0 = 0, nr1 = 0, nm0 = 0, nm1 = 0;
    Cursor cur{0, 0, 0};
    // the halves of the tile this row belongs to (warp-uniform): a block's keys
    // count for the row only if the row's query block kept it
    const int half_bit = pair ? (row < 64 ? 1 : 2) : 3;
    if (w < n_steps) fetch_blocks(cur, w, nr0, nr1, nm0, nm1);
    for (int j = w; j < n_steps && ok; j += 2, ++i) {
      int b0, b1;
      check_blocks(nr0, nr1, b0, b1);
      const int m0 = nm0, m1 = nm1;
      if (j + 2 < n_steps) fetch_blocks(cur, j + 2, nr0, nr1, nm0, nm1);
      // b < n_cand: at least one visible key
      const int n0 = (b0 >= 0 && (m0 & half_bit)) ? min(kBK, hi - b0 * kBK) : 0;
      const int n1 = (b1 >= 0 && (m1 & half_bit)) ? min(kBK, hi - b1 * kBK) : 0;
      const bool full = n0 == kBK && n1 == kBK;
      ok = tc::wait_warp(&bars[B_SFULL + w], i & 1, abort_flag, wait_ns);
      if (!ok) break;
      tc::fence_after_sync();
      float s[128];
      {
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld32p(tmem + lane_base + col_s + 32 * c, sr + 32 * c);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      }
      // S_w is in registers: the next QK of this pipeline may overwrite it
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[B_SFREE + w]);
      if (!full) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const bool valid = c < 64 ? (c < n0) : (c - 64 < n1);
          s[c] = valid ? s[c] : -INFINITY;
        }
      }
      float a0 = fmaxf(s[0], s[1]), a1 = fmaxf(s[2], s[3]), a2 = fmaxf(s[4], s[5]), a3 = fmaxf(s[6], s[7]);
#pragma unroll
      for (int c = 8; c < 128; c += 8) {
        a0 = max3(a0, s[c], s[c + 1]);
        a1 = max3(a1, s[c + 2], s[c + 3]);
        a2 = max3(a2, s[c + 4], s[c + 5]);
        a3 = max3(a3, s[c + 6], s[c + 7]);
      }
      const float mx = max3(a0, a1, fmaxf(a2, a3)) * scale_log2;
      bool rescale = false;
      float alpha = 1.f;
      if (i == 0) {
        m = mx;
      } else if (mx > m + 8.0f) {
        // the reference max grows by more than 2^8: move it and rescale O_w below
        alpha = (m == -INFINITY) ? 0.f : tc::ex2(m - mx);
        l *= alpha;
        m = mx;
        rescale = true;
      }
      // The previous PV of this pipeline frees the P buffer and leaves O_w quiescent.
      if (i > 0) {
        ok = tc::wait_warp(&bars[B_ODONE + w], (i - 1) & 1, abort_flag, wait_ns);
        if (!ok) break;
      }
      if (rescale) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16p(tmem + lane_base + col_o + 16 * c, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tc::tmem_st16p(tmem + lane_base + col_o + 16 * c, r);
        }
        tc::tmem_wait_st();
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      // P_j = 2^(s * scale - m) as bf16, written 8 keys (one 16-byte chunk) at a
      // time into the P buffer: [key half][128 rows][128 B], 128-byte swizzle
      const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-mref, -mref);
      uint64_t acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
      // One straight-line instance per case (no branch between the pairs, so
      // the independent exponentials interleave): full steps send a fixed share
      // of the pairs to the FMA pipe; steps with masked keys use MUFU only.
      auto write_p = [&](auto emu_tag) {
        constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * ch + e;  // key pair 2c, 2c+1
            float x0, x1, p0, p1;
            f2_split(fma2(f2(s[2 * c], s[2 * c + 1]), sc2, nm2), x0, x1);
            if (kEmu && (c & 15) >= 16 - kEmuPairs) {
              ex2_fma2(x0, x1, p0, p1);
            } else {
              p0 = tc::ex2(x0);  // 2^-inf = 0 on masked keys
              p1 = tc::ex2(x1);
            }
            if (e & 1) acc1 = add2(acc1, f2(p0, p1));
            else acc0 = add2(acc0, f2(p0, p1));
            pk[e] = pack_bf16(p0, p1);
          }
          *reinterpret_cast<uint4*>(pbuf + (ch / 8) * (kBQ * 128) + sw(row, ch % 8)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      };
      if (full) write_p(std::true_type{});
      else write_p(std::false_type{});
      {
        float r0, r1;
        f2_split(add2(acc0, acc1), r0, r1);
        l += r0 + r1;
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[B_PFULL + w]);
    }
    const int n_w = (n_steps - w + 1) / 2;  // steps of this pipeline
    if (ok && n_w > 0) ok = tc::wait_warp(&bars[B_ODONE + w], (n_w - 1) & 1, abort_flag, wait_ns);

    if (w == 1) {
      // hand (m, l) of the odd steps to the even group; O_1 stays in TMEM.
      // Fused form: q~ into S_1 (free: no QK follows) for the X MMA.
      if constexpr (FUSED) {
        if (ok) {
#pragma unroll
          for (int c = 0; c < R / 16; ++c) tc::tmem_st16p(tmem + lane_base + kColS1 + 16 * c, qt + 16 * c);
          tc::tmem_wait_st();
        }
      }
      merge_m[row] = (ok && n_w > 0) ? m : -INFINITY;
      merge_l[row] = (ok && n_w > 0) ? l : 0.f;
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[B_QTREADY]);
    } else {
      if (ok) ok = tc::wait_warp(&bars[B_QTREADY], 0, abort_flag, wait_ns);
      float gv = 0.f;
      if constexpr (FUSED) {
        const size_t rowi = (static_cast<size_t>(b) * P.L + tokc) * P.H + h;
        gv = __ldg(fa.gate + (P.gate_per_head ? rowi : rowi / P.H));
      }
      unsigned char* otile = pbuf;  // P_0 (free: the last even PV is done)
      if (ok) {
        tc::fence_after_sync();
        const float m1 = merge_m[row], l1 = merge_l[row];
        const float mm = fmaxf(m, m1);
        const float e0 = (m == -INFINITY) ? 0.f : tc::ex2(m - mm);
        const float e1 = (m1 == -INFINITY) ? 0.f : tc::ex2(m1 - mm);
        const bool has1 = l1 > 0.f;
        const float lt = l * e0 + (has1 ? l1 * e1 : 0.f);
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float c0 = e0 * inv, c1 = has1 ? e1 * inv : 0.f;
        if constexpr (!FUSED) {
          // log2 of the softmax denominator with the reference folded in: the
          // backward takes P = 2^(s * scale_log2 - lse) straight from it
          if (fa.lse != nullptr && tok < hi)
            fa.lse[(static_cast<size_t>(b) * P.L + tok) * P.H + h] = lt > 0.f ? mm + __log2f(lt) : INFINITY;
        }
        // O_s = (e0 O_0 + e1 O_1) / l for this row, in registers
        float o[D];
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t r0[16], r1[16];
          tc::tmem_ld16p(tmem + lane_base + kColO0 + 16 * c, r0);
          tc::tmem_ld16p(tmem + lane_base + kColO1 + 16 * c, r1);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o[16 * c + e] = has1 ? fmaf(__uint_as_float(r1[e]), c1, __uint_as_float(r0[e]) * c0)
                                 : __uint_as_float(r0[e]) * c0;
        }
        float coef = 0.f;
        if constexpr (FUSED) {
          float ss = 0.f;  // sum of squares of the O_s row (for r_i)
#pragma unroll
          for (int c = 0; c < D; ++c) ss = fmaf(o[c], o[c], ss);
          ok = tc::wait_warp(&bars[B_XFULL], 0, abort_flag, wait_ns);
          if (ok) {
            tc::fence_after_sync();
            float xs = 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tc::tmem_ld32(tmem + lane_base + kColS0 + 32 * c, r);
              tc::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) xs = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), xs);
            }
            coef = gv * sqrtf(ss / D) * rsqrtf(xs / D + P.rms_eps);
          }
        }
        if (ok) {
          // output row (bf16) into the output tile: [d half][128 rows][128 B], 128-byte swizzle
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            if constexpr (FUSED) {
              tc::tmem_ld32(tmem + lane_base + kColS0 + 32 * c, r);
              tc::tmem_wait_ld();
            }
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float ov = o[32 * c + 8 * q8 + e];
                if constexpr (FUSED) y[e] = fmaf(coef, __uint_as_float(r[8 * q8 + e]), ov);
                else y[e] = ov;
              }
              const uint4 v = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                         pack_bf16(y[6], y[7]));
              const int ch = 4 * c + q8;  // 16-byte chunk of the row (8 channels)
              *reinterpret_cast<uint4*>(otile + (ch / 8) * (kBQ * 128) + sw(row, ch % 8)) = v;
            }
          }
          tc::fence_proxy_async_smem();
        }
      }
      // every even-group thread reaches this barrier, whatever its verdict
      tc::named_barrier(1, 128);
      if (t128 == 0 && !*abort_flag) {
        for (int hf = 0; hf < S::kHalves; ++hf)
          tc::tma_store_4d(&tm_o, otile + hf * kBQ * 128, 64 * hf, h, q_row, q_slab);
        tc::bulk_commit_group();
        tc::bulk_wait_group_read0();
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*abort_flag) report_status(status, kStatusTimeout);
    if (*bad_flag) report_status(status, kStatusBadIndex);
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Time limit of the kernel's bounded waits on pipeline progress (the drain
// waits before TMEM is freed keep the 2 s limit whatever this says).
std::atomic<uint64_t> g_wait_limit_ns{tc::kWaitLimitNs};

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

// [B, L, H, d] bf16 as a 4-D tensor (d, H, L, B); box = 64 channels x `rows` tokens of one head.
// by_chunk: the same memory as (d, H, Tc, B * n_chunks), so that a query tile's
// loads stop (zero fill) and its stores are clipped at the end of its causal
// chunk (without a window Tc = L and the two views coincide).
bool make_map(CUtensorMap* map, const void* base, const Problem& P, int rows, bool by_chunk) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const int len = by_chunk ? P.chunk_tokens : P.L;
  const int slabs = by_chunk ? P.B * P.n_chunks : P.B;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(P.d), static_cast<cuuint64_t>(P.H),
                              static_cast<cuuint64_t>(len), static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(P.d) * 2, static_cast<cuuint64_t>(P.H) * P.d * 2,
                                 static_cast<cuuint64_t>(len) * P.H * P.d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// C^T head or tail, [B*H*n_chunks*d rows, r] bf16, as 128-byte rows (64 ranks;
// ranks past r read as zero) of d rows: one box per (batch, head, chunk).
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

template <int D, int R, bool FUSED, bool PAIR>
cudaError_t run_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* idx,
                   const FusedArgs& fa, uint16_t* o, unsigned* status, cudaStream_t stream) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;  // driver without cuTensorMapEncodeTiled
  // Q and O: 128-row boxes; K and V: 64-key boxes (one kept block)
  CUtensorMap mq, mk, mv, mo, mch, mcl;
  if (!make_map(&mq, q, P, kBQ, true) || !make_map(&mk, k, P, kBK, false) || !make_map(&mv, v, P, kBK, false) ||
      !make_map(&mo, o, P, kBQ, true))
    return cudaErrorInvalidValue;
  if (FUSED) {
    if (!make_ct_map(&mch, fa.ct_hi, P) || !make_ct_map(&mcl, fa.ct_lo, P)) return cudaErrorInvalidValue;
  } else {
    mch = mq;  // unused by the plain form
    mcl = mq;
  }
  const int smem = Smem<D, R, FUSED>::kTotal + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_attn_tc_kernel<D, R, FUSED, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits until the block's register pool can serve it: refuse
  // to launch a build whose per-thread allocation would leave it short.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, sparse_attn_tc_kernel<D, R, FUSED, PAIR>);
    if (e != cudaSuccess) return e;
    regs = attr.numRegs;
  }
  if (regs * kThreads < kRegsLow * 128 + kRegsHigh * 256) return cudaErrorInvalidConfiguration;
  // one CTA per 128-row query tile: a 128-row query block or a pair of 64-row ones
  const int tiles = P.block_q == 64 ? P.n_chunks * ((P.nq_chunk + 1) / 2) : P.n_qblk;
  const unsigned blocks = static_cast<unsigned>(P.B) * P.H * tiles;
  sparse_attn_tc_kernel<D, R, FUSED, PAIR><<<blocks, kThreads, smem, stream>>>(mq, mk, mv, mo, mch, mcl, P, idx, fa,
                                                                          status, g_wait_limit_ns.load());
  return cudaGetLastError();
}

}  // namespace

uint64_t set_attention_wait_limit(uint64_t limit_ns) { return g_wait_limit_ns.exchange(limit_ns); }

bool sparse_attn_tc_supported(const Problem& P) {
  return (P.block_q == kBQ || P.block_q == kBQ / 2) && P.block_k == kBK && (P.d == 64 || P.d == 128);
}

cudaError_t launch_sparse_attn_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const int32_t* block_idx, uint16_t* o_s, unsigned* status, cudaStream_t stream,
                                  float* lse) {
  const FusedArgs fa{nullptr, nullptr, nullptr, nullptr, nullptr, 0, lse};
  const bool pair = P.block_q == kBQ / 2;
  if (P.d == 128) return pair ? run_tc<128, 16, false, true>(P, q, k, v, block_idx, fa, o_s, status, stream)
                              : run_tc<128, 16, false, false>(P, q, k, v, block_idx, fa, o_s, status, stream);
  if (P.d == 64) return pair ? run_tc<64, 16, false, true>(P, q, k, v, block_idx, fa, o_s, status, stream)
                             : run_tc<64, 16, false, false>(P, q, k, v, block_idx, fa, o_s, status, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_sparse_attn_tc_fused(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                        const int32_t* block_idx, const uint16_t* p_q, const uint16_t* ct_hi,
                                        const uint16_t* ct_lo, const float2* rope_tab, const float* g, uint16_t* o,
                                        unsigned* status, cudaStream_t stream) {
  const FusedArgs fa{p_q, ct_hi, ct_lo, rope_tab, g, rope_table_entries(P), nullptr};
  const bool pair = P.block_q == kBQ / 2;
#define SDA_TC_FUSED(D_, R_)                                                                         \
  if (P.d == D_ && P.rank == R_)                                                                     \
    return pair ? run_tc<D_, R_, true, true>(P, q, k, v, block_idx, fa, o, status, stream)           \
                : run_tc<D_, R_, true, false>(P, q, k, v, block_idx, fa, o, status, stream);
  SDA_TC_FUSED(128, 16)
  SDA_TC_FUSED(128, 32)
  SDA_TC_FUSED(128, 64)
  SDA_TC_FUSED(64, 16)
  SDA_TC_FUSED(64, 32)
  SDA_TC_FUSED(64, 64)
#undef SDA_TC_FUSED
  return cudaErrorInvalidValue;
}

}  // namespace sda
