// Block-sparse attention A_M on the 5th-generation tensor cores (tcgen05),
// optionally with the low-rank readout and the gate fused into its epilogue
// (SparkDiffusion summary, robotworld.top, section 2.1: softmax(Q K^T /
// sqrt(d)) V restricted to the kept key blocks; O_lr = RMSNorm(q~^T C) with
// q~ = R_r(p) phi(P_q q); O = O_s + g r O_lr).
//
// One CTA per (batch, head, 128-row query block), 6 warps:
//   warp 0      TMA producer: Q once, then the kept key blocks two at a time
//               (a 128-key step) into a 2-stage K ring and a 2-stage V ring,
//               128-byte swizzled, no multicast;
//   warp 1      allocates 512 TMEM columns; one lane issues the MMAs:
//               S_j = Q K_j^T (M=128, N=128, K=d; operands from shared memory)
//               into one of two S buffers, and O += P_j V_j (A = P from TMEM,
//               B = V, MN-major) once the softmax has published P_j;
//   warps 2..5  softmax: thread = query row (TMEM lane), so the row max and
//               sum stay in registers. fp32 online softmax with exp2 and the
//               scale log2(e)/sqrt(d); the reference max moves (and O is
//               rescaled in TMEM) only when it grows by more than 2^8, which
//               is exact because numerator and denominator share it. P_j is
//               written as bf16 over the first 64 columns of S_j's buffer.
// TMEM: S0 cols [0,128), S1 [128,256), O [256, 256+d).
//
// Fused epilogue (sda_forward): the Q tile is still in shared memory, so
//   U = Q P_q^T            (M=128, N=r, K=d, bf16) into S0,
//   q~ = R_r(p) phi(U)     per thread (= per query row), written to S1 as fp32,
//   X = q~ C               (M=128, N=d, K=r, tf32, A from TMEM, C^T K-major in
//                           shared memory; r = 16 is zero-padded to 32) into S0,
// then O = O_s + g r X / sqrt(mean X^2 + eps), with O_s = O / l and r its RMS
// taken from the fp32 row. The standalone form writes O_s.
// Every wait is bounded (2 s); a CTA that gives up reports through the status
// word, drains its MMAs and TMA loads, frees TMEM and exits.

#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kThreads = 192;
constexpr int kBQ = 128;
constexpr int kBK = 64;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

template <int D, int R, bool FUSED>
struct Smem {
  static constexpr int kHalves = D / 64;                    // 64-element (128-byte) column slabs
  static constexpr int kQBytes = kHalves * kBQ * 128;        // [half][128 rows][128 B]
  static constexpr int kKVBytes = kHalves * 2 * kBK * 128;   // [half][128 keys][128 B]
  static constexpr int kPqBytes = FUSED ? kHalves * R * 128 : 0;   // P_q: [half][r rows][128 B]
  static constexpr int kRP = R < 32 ? 32 : R;                     // rank padded to whole 128-byte rows
  static constexpr int kCBytes = FUSED ? (kRP / 32) * D * 128 : 0;  // C^T: [r/32 slabs][d rows][128 B] fp32
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;                    // 2 stages
  static constexpr int kV = kK + 2 * kKVBytes;               // 2 stages
  static constexpr int kPq = kV + 2 * kKVBytes;
  static constexpr int kC = kPq + ((kPqBytes + 1023) / 1024) * 1024;
  static constexpr int kBars = kC + ((kCBytes + 1023) / 1024) * 1024;
  static constexpr int kTotal = kBars + 256;
};

// barrier slots
enum {
  B_Q = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7, B_SFULL = 9, B_PFULL = 11, B_ODONE = 13,
  B_DRAIN = 14, B_CONSTS = 15, B_UFULL = 16, B_QTFULL = 17, B_XFULL = 18, N_BARS = 19
};

struct FusedArgs {
  const uint16_t* p_q;    // [r, d] bf16
  const float* ct_state;  // [B, H, d, r] fp32 (C transposed)
  const float2* rope_tab; // cos/sin table (see common.cuh)
  const float* gate;      // [B, L] or [B, L, H]
};

template <int D, int R, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, Problem P, const int32_t* __restrict__ block_idx,
                      FusedArgs fa, uint16_t* __restrict__ out, unsigned* status) {
  using S = Smem<D, R, FUSED>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * N_BARS + 4);
  int* bad_flag = reinterpret_cast<int*>(smem + S::kBars + 8 * N_BARS + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int a = blockIdx.x % P.n_qblk;
  const int h = (blockIdx.x / P.n_qblk) % P.H;
  const int b = blockIdx.x / (P.n_qblk * P.H);
  const int keep = P.keep;
  const int n_steps = (keep + 1) / 2;
  const int32_t* idx = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * keep;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[B_KFULL + s], 1);
      tc::mbar_init(&bars[B_KEMPTY + s], 1);
      tc::mbar_init(&bars[B_VFULL + s], 1);
      tc::mbar_init(&bars[B_VEMPTY + s], 1);
      tc::mbar_init(&bars[B_SFULL + s], 1);
      tc::mbar_init(&bars[B_PFULL + s], 128);
    }
    tc::mbar_init(&bars[B_ODONE], 1);
    tc::mbar_init(&bars[B_DRAIN], 1);
    tc::mbar_init(&bars[B_CONSTS], 128);
    tc::mbar_init(&bars[B_UFULL], 1);
    tc::mbar_init(&bars[B_QTFULL], 128);
    tc::mbar_init(&bars[B_XFULL], 1);
    // A CTA of this launch (or an unread earlier one) gave up a wait: the
    // outputs are undefined until the status is read, so do no more work.
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    *bad_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
  }
  __syncthreads();
  if (*abort_flag) return;  // uniform: every thread reads the same shared flag
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // kept blocks of step j: (first, second); -1 marks an invalid block, -2 a missing one
  auto step_blocks = [&](int j, int& b0, int& b1) {
    b0 = __ldg(idx + 2 * j);
    b1 = (2 * j + 1 < keep) ? __ldg(idx + 2 * j + 1) : -2;
    if (b0 < 0 || b0 >= P.n_kblk) b0 = -1;
    if (b1 != -2 && (b1 < 0 || b1 >= P.n_kblk)) b1 = -1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      constexpr uint32_t kHalfBytes = kBK * 128;  // one 64-key x 64-element box
      bool ok = true;
      tc::mbar_arrive_expect_tx(&bars[B_Q], S::kQBytes);
      for (int hf = 0; hf < S::kHalves; ++hf)
        tc::tma_load_4d(smem + S::kQ + hf * kBQ * 128, &tm_q, &bars[B_Q], 64 * hf, h, a * kBQ, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_steps && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int b0, b1;
        step_blocks(j, b0, b1);
        if (b0 == -1 || b1 == -1) *bad_flag = 1;
        const int lb0 = b0 >= 0 ? b0 : 0;
        const int lb1 = b1 >= 0 ? b1 : lb0;  // missing / invalid second block: reload one, masked
        unsigned char* kst = smem + S::kK + st * S::kKVBytes;
        unsigned char* vst = smem + S::kV + st * S::kKVBytes;
        ok = tc::wait1(&bars[B_KEMPTY + st], ph ^ 1, abort_flag);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&bars[B_KFULL + st], S::kKVBytes);
        for (int hf = 0; hf < S::kHalves; ++hf) {
          tc::tma_load_4d(kst + hf * 2 * kHalfBytes, &tm_k, &bars[B_KFULL + st], 64 * hf, h, lb0 * kBK, b);
          tc::tma_load_4d(kst + hf * 2 * kHalfBytes + kHalfBytes, &tm_k, &bars[B_KFULL + st], 64 * hf, h, lb1 * kBK, b);
        }
        k_issued = j + 1;
        ok = tc::wait1(&bars[B_VEMPTY + st], ph ^ 1, abort_flag);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&bars[B_VFULL + st], S::kKVBytes);
        for (int hf = 0; hf < S::kHalves; ++hf) {
          tc::tma_load_4d(vst + hf * 2 * kHalfBytes, &tm_v, &bars[B_VFULL + st], 64 * hf, h, lb0 * kBK, b);
          tc::tma_load_4d(vst + hf * 2 * kHalfBytes + kHalfBytes, &tm_v, &bars[B_VFULL + st], 64 * hf, h, lb1 * kBK, b);
        }
        v_issued = j + 1;
      }
      // Drain: make sure every load this thread issued has landed before exit.
      volatile int never = 0;
      tc::wait1(&bars[B_Q], 0, &never);
      for (int j = k_issued - 2 < 0 ? 0 : k_issued - 2; j < k_issued; ++j)
        tc::wait1(&bars[B_KFULL + (j & 1)], (j >> 1) & 1, &never);
      for (int j = v_issued - 2 < 0 ? 0 : v_issued - 2; j < v_issued; ++j)
        tc::wait1(&bars[B_VFULL + (j & 1)], (j >> 1) & 1, &never);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(128, 128, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, D, true);
      bool ok = tc::wait1(&bars[B_Q], 0, abort_flag);
      if (ok) tc::fence_after_sync();
      for (int j = 0; j <= n_steps && ok; ++j) {
        if (j < n_steps) {
          const int st = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          ok = tc::wait1(&bars[B_KFULL + st], ph, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* kst = smem + S::kK + st * S::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hf = kk / 4, w = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(smem + S::kQ + hf * kBQ * 128 + w * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(kst + hf * 2 * kBK * 128 + w * 32, 16, 1024);
            tc::mma_ss(tmem + (st ? kColS1 : kColS0), da, db, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[B_SFULL + st]);
          tc::commit(&bars[B_KEMPTY + st]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj & 1;
          const uint32_t ph = (jj >> 1) & 1;
          ok = tc::wait1(&bars[B_PFULL + st], ph, abort_flag);
          if (ok) ok = tc::wait1(&bars[B_VFULL + st], ph, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* vst = smem + S::kV + st * S::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < 2 * kBK / 16; ++kk) {
            // 16 keys per MMA: rows kk*16.. of the V stage; the d slabs are 16 KB apart (LBO)
            const uint64_t db = tc::smem_desc_sw128(vst + kk * 16 * 128, 2 * kBK * 128, 1024);
            tc::mma_ts(tmem + kColO, tmem + (st ? kColS1 : kColS0) + kk * 8, db, idesc_pv,
                       (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(&bars[B_VEMPTY + st]);
          tc::commit(&bars[B_ODONE]);
        }
      }
      if constexpr (FUSED) {
        // U = Q P_q^T into S0 (issued after the last PV, so after every read of S0)
        if (ok) ok = tc::wait1(&bars[B_CONSTS], 0, abort_flag);
        if (ok) {
          tc::fence_after_sync();
          constexpr uint32_t idesc_u = tc::idesc_bf16(128, R, false);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hf = kk / 4, w = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(smem + S::kQ + hf * kBQ * 128 + w * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(smem + S::kPq + hf * R * 128 + w * 32, 16, 1024);
            tc::mma_ss(tmem + kColS0, da, db, idesc_u, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[B_UFULL]);
          // X = q~ C into S0 once the features are in S1 (tf32, 8 ranks per MMA)
          ok = tc::wait1(&bars[B_QTFULL], 0, abort_flag);
        }
        if (ok) {
          tc::fence_after_sync();
          constexpr uint32_t idesc_x = tc::idesc_tf32(128, D, false);
#pragma unroll
          for (int kk = 0; kk < S::kRP / 8; ++kk) {
            // 8 ranks (32 bytes) per MMA inside a 128-byte row; 32-rank slabs of d rows
            const uint64_t db = tc::smem_desc_sw128(smem + S::kC + (kk / 4) * D * 128 + (kk % 4) * 32, 16, 1024);
            tc::mma_ts_tf32(tmem + kColS0, tmem + kColS1 + kk * 8, db, idesc_x, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[B_XFULL]);
        }
      }
      // every MMA issued above has retired once the drain barrier flips
      tc::commit(&bars[B_DRAIN]);
      volatile int never = 0;
      tc::wait1(&bars[B_DRAIN], 0, &never);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;                 // TMEM lanes [32*quarter, +32)
    const int row = 32 * quarter + lane;          // query row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const size_t bh = static_cast<size_t>(b) * P.H + h;

    if constexpr (FUSED) {
      // P_q (bf16, K-major, 128-byte swizzle) and C (fp32, MN-major, 128-byte
      // swizzle) into shared memory for the epilogue MMAs.
      const int t = threadIdx.x - 64;  // 0..127
      for (int e = t; e < R * (D / 8); e += 128) {
        const int n = e / (D / 8), c8 = e % (D / 8);  // row n, 16-byte chunk c8 (8 channels)
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(fa.p_q + n * D) + c8);
        *reinterpret_cast<uint4*>(smem + S::kPq + (c8 / 8) * R * 128 + tc::sw128_offset(n, c8 % 8)) = v;
      }
      // C^T rows (d of them, r fp32 each); ranks past r (r = 16 only) are zero
      const float* cs = fa.ct_state + bh * R * D;
      for (int e = t; e < D * (S::kRP / 4); e += 128) {
        const int n = e / (S::kRP / 4), c4 = e % (S::kRP / 4);  // channel n, ranks 4*c4..
        const float4 v = (4 * c4 < R) ? __ldg(reinterpret_cast<const float4*>(cs + n * R) + c4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(smem + S::kC + (c4 / 8) * D * 128 + tc::sw128_offset(n, c4 % 8)) = v;
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_CONSTS]);
    }

    float m = -INFINITY;  // reference max (log2 units)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_steps && ok; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      int b0, b1;
      step_blocks(j, b0, b1);
      const int n0 = b0 >= 0 ? min(kBK, P.L - b0 * kBK) : 0;
      const int n1 = b1 >= 0 ? min(kBK, P.L - b1 * kBK) : 0;
      ok = tc::wait_warp(&bars[B_SFULL + st], ph, abort_flag);
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t s_addr = tmem + lane_base + (st ? kColS1 : kColS0);
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32p(s_addr + 32 * c, sr + 32 * c);
      tc::tmem_wait_ld();
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      float mx = -INFINITY;
      if (n0 == kBK && n1 == kBK) {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx = fmaxf(mx, s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const bool valid = c < 64 ? (c < n0) : (c - 64 < n1);
          s[c] = valid ? s[c] : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      }
      mx *= scale_log2;
      if (j == 0) {
        m = mx;
      } else if (mx > m + 8.0f) {
        // the reference max grows by more than 2^8: rescale O (PV_{j-1} must be done)
        ok = tc::wait_warp(&bars[B_ODONE], (j - 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const float alpha = (m == -INFINITY) ? 0.f : tc::ex2(m - mx);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tc::tmem_ld32(tmem + lane_base + kColO + 32 * c, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tc::tmem_st32(tmem + lane_base + kColO + 32 * c, r);
        }
        tc::tmem_wait_st();
        l *= alpha;
        m = mx;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      float rs = 0.f;
      // P_j as bf16 pairs over the first 64 columns of S_j's buffer (all of
      // S_j is already in registers): keys 2c, 2c+1 -> column c.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = tc::ex2(fmaf(s[64 * half + 2 * c], scale_log2, -mref));
          const float p1 = tc::ex2(fmaf(s[64 * half + 2 * c + 1], scale_log2, -mref));
          rs += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
        tc::tmem_st32(s_addr + 32 * half, pk);
      }
      l += rs;
      tc::tmem_wait_st();
      // PV_{j-1} must have retired before P_j is published (keeps the
      // O-done phases one step apart, which the parity waits rely on)
      if (j >= 1) {
        ok = tc::wait_warp(&bars[B_ODONE], (j - 1) & 1, abort_flag);
        if (!ok) break;
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[B_PFULL + st]);
    }
    if (ok) ok = tc::wait_warp(&bars[B_ODONE], (n_steps - 1) & 1, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      float o[D];
      {
        uint32_t orr[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tc::tmem_ld32p(tmem + lane_base + kColO + 32 * c, orr + 32 * c);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] = __uint_as_float(orr[c]);
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        o[c] *= inv;
        ss += o[c] * o[c];
      }
      const int tok = a * kBQ + row;
      const int tokc = tok < P.L ? tok : P.L - 1;
      const size_t rowi = (static_cast<size_t>(b) * P.L + tokc) * P.H + h;
      uint4* dst = reinterpret_cast<uint4*>(out + rowi * D);
      if constexpr (FUSED) {
        // q~ = R_r(p) phi(U) for this row, into S1 as fp32
        ok = tc::wait_warp(&bars[B_UFULL], 0, abort_flag);
        if (ok) {
          tc::fence_after_sync();
          uint32_t ur[R];
#pragma unroll
          for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(tmem + lane_base + kColS0 + 16 * c, ur + 16 * c);
          tc::tmem_wait_ld();
          const int w = tokc % P.grid_w;
          const int hh = (tokc / P.grid_w) % P.grid_h;
          const int tt = tokc / (P.grid_w * P.grid_h);
          // table rows of this token per axis, indexed by the global pair number
          const float2* tab_t = fa.rope_tab + tt * P.pairs_t;
          const float2* tab_h = fa.rope_tab + P.grid_t * P.pairs_t + hh * P.pairs_h - P.pairs_t;
          const float2* tab_w =
              fa.rope_tab + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + w * P.pairs_w - P.pairs_t - P.pairs_h;
#pragma unroll
          for (int mm = 0; mm < R / 2; ++mm) {
            const float x = elu_plus_one(__uint_as_float(ur[2 * mm]));
            const float y = elu_plus_one(__uint_as_float(ur[2 * mm + 1]));
            const float2* src = mm < P.pairs_t ? tab_t : (mm < P.pairs_t + P.pairs_h ? tab_h : tab_w);
            const float2 cs2 = __ldg(src + mm);
            ur[2 * mm] = __float_as_uint(x * cs2.x - y * cs2.y);
            ur[2 * mm + 1] = __float_as_uint(x * cs2.y + y * cs2.x);
          }
#pragma unroll
          for (int c = 0; c < R / 16; ++c) tc::tmem_st16p(tmem + lane_base + kColS1 + 16 * c, ur + 16 * c);
          if constexpr (R < S::kRP) {
            uint32_t zero[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
            for (int c = R / 16; c < S::kRP / 16; ++c) tc::tmem_st16p(tmem + lane_base + kColS1 + 16 * c, zero);
          }
          tc::tmem_wait_st();
          tc::fence_before_sync();
          tc::mbar_arrive(&bars[B_QTFULL]);
          ok = tc::wait_warp(&bars[B_XFULL], 0, abort_flag);
        }
        if (ok) {
          tc::fence_after_sync();
          // X row: RMS first, then the fused output
          float xs = 0.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tc::tmem_ld32(tmem + lane_base + kColS0 + 32 * c, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) xs += __uint_as_float(r[e]) * __uint_as_float(r[e]);
          }
          const float gv = __ldg(fa.gate + (P.gate_per_head ? rowi : rowi / P.H));
          const float coef = gv * sqrtf(ss / D) * rsqrtf(xs / D + P.rms_eps);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tc::tmem_ld32(tmem + lane_base + kColS0 + 32 * c, r);
            tc::tmem_wait_ld();
            if (tok < P.L) {
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) {
                const int c0 = 32 * c + 8 * q8;
                uint4 y;
                y.x = pack_bf16(fmaf(coef, __uint_as_float(r[8 * q8 + 0]), o[c0 + 0]),
                                fmaf(coef, __uint_as_float(r[8 * q8 + 1]), o[c0 + 1]));
                y.y = pack_bf16(fmaf(coef, __uint_as_float(r[8 * q8 + 2]), o[c0 + 2]),
                                fmaf(coef, __uint_as_float(r[8 * q8 + 3]), o[c0 + 3]));
                y.z = pack_bf16(fmaf(coef, __uint_as_float(r[8 * q8 + 4]), o[c0 + 4]),
                                fmaf(coef, __uint_as_float(r[8 * q8 + 5]), o[c0 + 5]));
                y.w = pack_bf16(fmaf(coef, __uint_as_float(r[8 * q8 + 6]), o[c0 + 6]),
                                fmaf(coef, __uint_as_float(r[8 * q8 + 7]), o[c0 + 7]));
                dst[c0 / 8] = y;
              }
            }
          }
        }
      } else {
        if (tok < P.L) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            uint4 y;
            y.x = pack_bf16(o[8 * c + 0], o[8 * c + 1]);
            y.y = pack_bf16(o[8 * c + 2], o[8 * c + 3]);
            y.z = pack_bf16(o[8 * c + 4], o[8 * c + 5]);
            y.w = pack_bf16(o[8 * c + 6], o[8 * c + 7]);
            dst[c] = y;
          }
        }
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

template <int D, int R, bool FUSED>
cudaError_t run_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* idx,
                   const FusedArgs& fa, uint16_t* o, unsigned* status, cudaStream_t stream) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;  // driver without cuTensorMapEncodeTiled
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, P, kBQ) || !make_map(&mk, k, P, kBK) || !make_map(&mv, v, P, kBK))
    return cudaErrorInvalidValue;
  const int smem = Smem<D, R, FUSED>::kTotal + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_attn_tc_kernel<D, R, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>(P.B) * P.H * P.n_qblk;
  sparse_attn_tc_kernel<D, R, FUSED><<<blocks, kThreads, smem, stream>>>(mq, mk, mv, P, idx, fa, o, status);
  return cudaGetLastError();
}

}  // namespace

bool sparse_attn_tc_supported(const Problem& P) {
  return P.block_q == kBQ && P.block_k == kBK && (P.d == 64 || P.d == 128);
}

cudaError_t launch_sparse_attn_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const int32_t* block_idx, uint16_t* o_s, unsigned* status, cudaStream_t stream) {
  const FusedArgs fa{nullptr, nullptr, nullptr, nullptr};
  if (P.d == 128) return run_tc<128, 16, false>(P, q, k, v, block_idx, fa, o_s, status, stream);
  if (P.d == 64) return run_tc<64, 16, false>(P, q, k, v, block_idx, fa, o_s, status, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_sparse_attn_tc_fused(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                        const int32_t* block_idx, const uint16_t* p_q, const float* ct_state,
                                        const float2* rope_tab, const float* g, uint16_t* o, unsigned* status,
                                        cudaStream_t stream) {
  const FusedArgs fa{p_q, ct_state, rope_tab, g};
#define SDA_TC_FUSED(D_, R_) \
  if (P.d == D_ && P.rank == R_) return run_tc<D_, R_, true>(P, q, k, v, block_idx, fa, o, status, stream);
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
