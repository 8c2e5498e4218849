// Backward of the block-sparse attention A_M on the tensor cores (tcgen05):
// the gradients dq, dk, dv of sum(O_s . dO_s) for O_s = softmax(Q K^T /
// sqrt(d)) V over the kept key blocks (SparkDiffusion summary, robotworld.top,
// section 2.1; the training path that needs it: H3 portability report,
// sections 2.1-2.2). With P the softmax of a query row over its kept keys,
// D_i = dO_s,i . O_s,i and dP = dO_s V^T:
//   dS = P (dP - D) / sqrt(d),   dq = dS K,   dk = dS^T Q,   dv = P^T dO_s.
// P comes back exactly from the forward's log2-sum-exp (lse): P = 2^(s c - lse)
// with s = q . k and c = log2(e) / sqrt(d).
//
// Kernel 1 (dq): one CTA per (batch, head, 128-row query block), walking its
// kept 64-key blocks in map order. Per block j: S_j = Q K_j^T and dP_j =
// dO_s V_j^T (M = 128, N = 64) into double-buffered TMEM; the compute
// warpgroup (thread = query row) forms dS_j as bf16 in shared memory; dQ +=
// dS_j K_j (M = 128, N = d, K = 64, K_j read MN-major) accumulates in TMEM.
// Warps: 0 S issuer (TMEM owner), 1 dP issuer, 2 dQ issuer, 3 TMA loader
// (Q and dO_s once, a 3-stage K ring and a 2-stage V ring), 4..7 compute.
//
// Kernel 2 (dk, dv): one CTA per (batch, head, 64-key block), walking the
// query blocks that kept it (the transposed map, ascending). Per query block
// i: S_i = Q_i K^T and dP_i = dO_s,i V^T (M = 128 rows, N = 64 keys) into
// double-buffered TMEM; the compute warpgroup forms P_i and dS_i as bf16 in
// shared memory; dV^T += dO_s,i^T P_i and dK^T += Q_i^T dS_i (M = d = 128, N =
// 64 keys, K = 128 rows; both operands read MN-major from the row tiles), so
// no M = 64 accumulator is needed. Warps: 0 TMA loader (K, V once; 2-stage Q
// and dO_s rings), 1 S issuer (TMEM owner), 2 dP issuer, 3 dV issuer, 4..7
// compute, 8 dK issuer.
//
// Both kernels add into dq / dk / dv (which already hold the low-rank
// branch's part) in a fixed order per element: reruns are bit-identical.
// Keys past L and query rows past L are masked to P = 0. A map entry outside
// [0, N_kblk) is treated as a fully masked block and reported through the
// status word. Every wait is bounded (2 s); a CTA that gives up reports it,
// drains its loads and MMAs, frees TMEM and exits.

#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kBQ = 128;
constexpr int kBK = 64;
constexpr int kD = 128;          // head dim of the tensor-core backward
constexpr int kHalves = kD / 64;  // 64-channel (128-byte) slabs of a row
constexpr uint32_t kTmemCols = 512;

// ---------------------------------------------------------------------------
// dq kernel
// ---------------------------------------------------------------------------

constexpr int kDqThreads = 256;
constexpr int kKStages = 3, kVStages = 2;
// TMEM columns: S_0, S_1, dP_0, dP_1 (64 each), dQ (d)
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;

struct DqSmem {
  static constexpr int kQBytes = kHalves * kBQ * 128;   // [half][128 rows][128 B]
  static constexpr int kKVBytes = kHalves * kBK * 128;  // [half][64 keys][128 B]
  static constexpr int kDSBytes = kBQ * 128;            // [128 rows][64 keys] bf16
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kQBytes;
  static constexpr int kK = kDO + kQBytes;
  static constexpr int kV = kK + kKStages * kKVBytes;
  static constexpr int kDS = kV + kVStages * kKVBytes;
  static constexpr int kBars = kDS + 2 * kDSBytes;
  static constexpr int kTotal = kBars + 256;
};

enum {
  DQ_QFULL = 0, DQ_DOFULL = 1, DQ_KFULL = 2, DQ_KFREE = 5, DQ_VFULL = 8, DQ_VFREE = 10, DQ_SFULL = 12,
  DQ_DPFULL = 14, DQ_SFREE = 16, DQ_DSFULL = 18, DQ_DSFREE = 20, DQ_DRAIN = 22, DQ_NBARS = 26
};

__device__ __forceinline__ uint32_t sw(uint32_t row, uint32_t chunk) { return tc::sw128_offset(row, chunk); }

// The kept block of slot j of a map row: the index, or -1 when it lies outside [0, N_kblk).
__device__ __forceinline__ int kept(const Problem& P, const int32_t* row, int j) {
  const int kb = __ldg(row + j);
  return (kb >= 0 && kb < P.n_kblk) ? kb : -1;
}

__global__ void __launch_bounds__(kDqThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Problem P,
                 const int32_t* __restrict__ block_idx, const float* __restrict__ lse, const float* __restrict__ dd,
                 float* __restrict__ dq, unsigned* status) {
  using S = DqSmem;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * DQ_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * DQ_NBARS + 4);
  int* bad_flag = reinterpret_cast<int*>(smem + S::kBars + 8 * DQ_NBARS + 8);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int a = blockIdx.x % P.n_qblk;
  const int h = (blockIdx.x / P.n_qblk) % P.H;
  const int b = blockIdx.x / (P.n_qblk * P.H);
  const int n = P.keep;  // kept blocks of this query block, one 64-key step each
  const int32_t* idx = block_idx + ((static_cast<size_t>(b) * P.H + h) * P.n_qblk + a) * P.keep;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars[DQ_QFULL], 1);
    tc::mbar_init(&bars[DQ_DOFULL], 1);
    for (int s = 0; s < kKStages; ++s) {
      tc::mbar_init(&bars[DQ_KFULL + s], 1);
      tc::mbar_init(&bars[DQ_KFREE + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[DQ_VFULL + s], 1);
      tc::mbar_init(&bars[DQ_VFREE + s], 1);
      tc::mbar_init(&bars[DQ_SFULL + s], 1);
      tc::mbar_init(&bars[DQ_DPFULL + s], 1);
      tc::mbar_init(&bars[DQ_SFREE + s], 128);
      tc::mbar_init(&bars[DQ_DSFULL + s], 128);
      tc::mbar_init(&bars[DQ_DSFREE + s], 1);
    }
    for (int r = 0; r < 4; ++r) tc::mbar_init(&bars[DQ_DRAIN + r], 1);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    *bad_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
    tc::tma_prefetch(&tm_do);
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
  }
  __syncthreads();
  if (*abort_flag) return;  // uniform: every thread reads the same shared flag
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    if (lane == 0) {
      volatile int never = 0;
      bool ok = true;
      if (warp == 3) {
        // ------------------------------------------------------------ TMA loader
        constexpr uint32_t kHalfBytes = kBK * 128;
        tc::mbar_arrive_expect_tx(&bars[DQ_QFULL], S::kQBytes);
        tc::mbar_arrive_expect_tx(&bars[DQ_DOFULL], S::kQBytes);
        for (int hf = 0; hf < kHalves; ++hf) {
          tc::tma_load_4d(smem + S::kQ + hf * kBQ * 128, &tm_q, &bars[DQ_QFULL], 64 * hf, h, a * kBQ, b);
          tc::tma_load_4d(smem + S::kDO + hf * kBQ * 128, &tm_do, &bars[DQ_DOFULL], 64 * hf, h, a * kBQ, b);
        }
        int k_loaded = 0, v_loaded = 0;  // loads issued (each one is waited for below)
        for (int j = 0; j < n && ok; ++j) {
          int kb = kept(P, idx, j);
          if (kb < 0) {
            *bad_flag = 1;
            kb = 0;  // a fully masked block keeps the pipeline's shape
          }
          const int ks = j % kKStages, vs = j % kVStages;
          if (j >= kKStages) ok = tc::wait1(&bars[DQ_KFREE + ks], ((j / kKStages) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&bars[DQ_KFULL + ks], S::kKVBytes);
          for (int hf = 0; hf < kHalves; ++hf)
            tc::tma_load_4d(smem + S::kK + ks * S::kKVBytes + hf * kHalfBytes, &tm_k, &bars[DQ_KFULL + ks], 64 * hf,
                            h, kb * kBK, b);
          ++k_loaded;
          if (j >= kVStages) ok = tc::wait1(&bars[DQ_VFREE + vs], ((j / kVStages) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&bars[DQ_VFULL + vs], S::kKVBytes);
          for (int hf = 0; hf < kHalves; ++hf)
            tc::tma_load_4d(smem + S::kV + vs * S::kKVBytes + hf * kHalfBytes, &tm_v, &bars[DQ_VFULL + vs], 64 * hf,
                            h, kb * kBK, b);
          ++v_loaded;
        }
        // drain: every load issued has landed before the CTA can exit
        tc::wait1(&bars[DQ_QFULL], 0, &never);
        tc::wait1(&bars[DQ_DOFULL], 0, &never);
        for (int j = (k_loaded > kKStages ? k_loaded - kKStages : 0); j < k_loaded; ++j)
          tc::wait1(&bars[DQ_KFULL + j % kKStages], (j / kKStages) & 1, &never);
        for (int j = (v_loaded > kVStages ? v_loaded - kVStages : 0); j < v_loaded; ++j)
          tc::wait1(&bars[DQ_VFULL + j % kVStages], (j / kVStages) & 1, &never);
      } else if (warp < 2) {
        // ------------------------------------------------ S (warp 0) / dP (warp 1) issuer
        const bool is_s = warp == 0;
        constexpr uint32_t idesc = tc::idesc_bf16(128, kBK, false);
        const unsigned char* a_tile = smem + (is_s ? S::kQ : S::kDO);
        ok = tc::wait1(&bars[is_s ? DQ_QFULL : DQ_DOFULL], 0, abort_flag);
        for (int j = 0; j < n && ok; ++j) {
          const int buf = j & 1;
          if (is_s) ok = tc::wait1(&bars[DQ_KFULL + j % kKStages], (j / kKStages) & 1, abort_flag);
          else ok = tc::wait1(&bars[DQ_VFULL + j % kVStages], (j / kVStages) & 1, abort_flag);
          // the compute warps have read S / dP of step j - 2 out of this buffer
          if (ok && j >= 2) ok = tc::wait1(&bars[DQ_SFREE + buf], ((j >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* b_tile =
              is_s ? smem + S::kK + (j % kKStages) * S::kKVBytes : smem + S::kV + (j % kVStages) * S::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int hf = kk / 4, c = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(a_tile + hf * kBQ * 128 + c * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(b_tile + hf * kBK * 128 + c * 32, 16, 1024);
            tc::mma_ss(tmem + (is_s ? kColS : kColDP) + buf * kBK, da, db, idesc, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[(is_s ? DQ_SFULL : DQ_DPFULL) + buf]);
          if (!is_s) tc::commit(&bars[DQ_VFREE + j % kVStages]);  // V_j is read only here
        }
      } else if (warp == 2) {
        // ---------------------------------------------------------- dQ issuer
        constexpr uint32_t idesc = tc::idesc_bf16(128, kD, true);  // A = dS K-major, B = K MN-major
        for (int j = 0; j < n && ok; ++j) {
          const int buf = j & 1;
          ok = tc::wait1(&bars[DQ_DSFULL + buf], (j >> 1) & 1, abort_flag);
          if (ok) ok = tc::wait1(&bars[DQ_KFULL + j % kKStages], (j / kKStages) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* ds = smem + S::kDS + buf * S::kDSBytes;
          const unsigned char* kt = smem + S::kK + (j % kKStages) * S::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t da = tc::smem_desc_sw128(ds + kk * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(kt + kk * 16 * 128, kBK * 128, 1024);
            tc::mma_ss(tmem + kColDQ, da, db, idesc, (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(&bars[DQ_DSFREE + buf]);
          tc::commit(&bars[DQ_KFREE + j % kKStages]);  // S_j (earlier) and dQ_j were its readers
        }
      }
      // every MMA this thread issued has completed before TMEM can be freed
      if (warp < 3) {
        tc::commit(&bars[DQ_DRAIN + warp]);
        tc::wait1(&bars[DQ_DRAIN + warp], 0, &never);
      }
    }
  } else {
    // -------------------------------------------------------------- compute
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    const int tok = a * kBQ + row;
    const bool row_ok = tok < P.L;
    const size_t rowi = (static_cast<size_t>(b) * P.L + (row_ok ? tok : 0)) * P.H + h;
    const float lse2 = row_ok ? __ldg(lse + rowi) : 0.f;
    const float dsum = row_ok ? __ldg(dd + rowi) : 0.f;
    const float c2 = 1.4426950408889634f / sqrtf(static_cast<float>(kD));  // log2(e) / sqrt(d)
    const float sd = 1.f / sqrtf(static_cast<float>(kD));
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int buf = j & 1;
      const int kb = kept(P, idx, j);
      const int nk = (kb < 0 || !row_ok) ? 0 : min(kBK, P.L - kb * kBK);  // valid keys of this block
      ok = tc::wait_warp(&bars[DQ_SFULL + buf], (j >> 1) & 1, abort_flag);
      if (ok) ok = tc::wait_warp(&bars[DQ_DPFULL + buf], (j >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::fence_after_sync();
      uint32_t sr[kBK], pr[kBK];
      tc::tmem_ld32p(tmem + lane_base + kColS + buf * kBK, sr);
      tc::tmem_ld32p(tmem + lane_base + kColS + buf * kBK + 32, sr + 32);
      tc::tmem_ld32p(tmem + lane_base + kColDP + buf * kBK, pr);
      tc::tmem_ld32p(tmem + lane_base + kColDP + buf * kBK + 32, pr + 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[DQ_SFREE + buf]);
      // dS of step j - 2 has been consumed by its dQ MMAs: the buffer is free
      if (j >= 2) {
        ok = tc::wait_warp(&bars[DQ_DSFREE + buf], ((j >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
      }
      unsigned char* ds = smem + S::kDS + buf * S::kDSBytes;
#pragma unroll
      for (int ch = 0; ch < kBK / 8; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * ch + 2 * e;
          float v[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float p = (c + u < nk) ? tc::ex2(__uint_as_float(sr[c + u]) * c2 - lse2) : 0.f;
            v[u] = p * (__uint_as_float(pr[c + u]) - dsum) * sd;
          }
          pk[e] = pack_bf16(v[0], v[1]);
        }
        *reinterpret_cast<uint4*>(ds + sw(row, ch)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[DQ_DSFULL + buf]);
    }
    // the last dQ MMAs have completed: add this row of dQ to dq
    if (ok && n > 0) ok = tc::wait_warp(&bars[DQ_DSFREE + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort_flag);
    if (ok) {
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + lane_base + kColDQ + 32 * c, r);
        tc::tmem_wait_ld();
        if (row_ok) {
          // all loads first, then the stores: the 8 round trips overlap
          float4* dst = reinterpret_cast<float4*>(dq + rowi * kD + 32 * c);
          float4 x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = dst[e];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e].x += __uint_as_float(r[4 * e]);
            x[e].y += __uint_as_float(r[4 * e + 1]);
            x[e].z += __uint_as_float(r[4 * e + 2]);
            x[e].w += __uint_as_float(r[4 * e + 3]);
            dst[e] = x[e];
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
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dk / dv kernel
// ---------------------------------------------------------------------------

constexpr int kKvThreads = 288;  // 9 warps
// TMEM columns: S_0, S_1, dP_0, dP_1 (64 each), dV^T, dK^T (64 keys each; lanes = channels)
constexpr uint32_t kColDV = 256, kColDK = 320;

struct KvSmem {
  static constexpr int kRowBytes = kHalves * kBQ * 128;  // a 128-row tile of Q or dO_s
  static constexpr int kKeyBytes = kHalves * kBK * 128;  // the 64-key tile of K or V
  static constexpr int kPBytes = kBQ * 128;              // [128 rows][64 keys] bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKeyBytes;
  static constexpr int kQ = kV + kKeyBytes;               // 2 stages
  static constexpr int kDO = kQ + 2 * kRowBytes;          // 2 stages
  static constexpr int kP = kDO + 2 * kRowBytes;
  static constexpr int kDS = kP + kPBytes;
  static constexpr int kBars = kDS + kPBytes;
  static constexpr int kTotal = kBars + 256;
};

enum {
  KV_KVFULL = 0, KV_QFULL = 1, KV_QFREE = 3, KV_DOFULL = 5, KV_DOFREE = 7, KV_SFULL = 9, KV_DPFULL = 11,
  KV_SFREE = 13, KV_PFULL = 15, KV_PFREE = 16, KV_DSFULL = 17, KV_DSFREE = 18, KV_DRAIN = 19, KV_NBARS = 24
};

__global__ void __launch_bounds__(kKvThreads, 1)
bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Problem P,
                  const int32_t* __restrict__ offs, const int32_t* __restrict__ list, const float* __restrict__ lse,
                  const float* __restrict__ dd, float* __restrict__ dk, float* __restrict__ dv, unsigned* status) {
  using S = KvSmem;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * KV_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * KV_NBARS + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kb = blockIdx.x % P.n_kblk;
  const int h = (blockIdx.x / P.n_kblk) % P.H;
  const int b = blockIdx.x / (P.n_kblk * P.H);
  const long long bh = static_cast<long long>(b) * P.H + h;
  const int32_t* o = offs + bh * (P.n_kblk + 1);
  const int x0 = __ldg(o + kb), n = __ldg(o + kb + 1) - x0;  // query blocks that kept this key block
  const int32_t* qb = list + bh * static_cast<long long>(P.n_qblk) * P.keep + x0;
  if (n == 0) return;  // no attention gradient reaches this key block (uniform exit)

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars[KV_KVFULL], 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[KV_QFULL + s], 1);
      tc::mbar_init(&bars[KV_QFREE + s], 1);
      tc::mbar_init(&bars[KV_DOFULL + s], 1);
      tc::mbar_init(&bars[KV_DOFREE + s], 1);
      tc::mbar_init(&bars[KV_SFULL + s], 1);
      tc::mbar_init(&bars[KV_DPFULL + s], 1);
      tc::mbar_init(&bars[KV_SFREE + s], 128);
    }
    tc::mbar_init(&bars[KV_PFULL], 128);
    tc::mbar_init(&bars[KV_PFREE], 1);
    tc::mbar_init(&bars[KV_DSFULL], 128);
    tc::mbar_init(&bars[KV_DSFREE], 1);
    for (int r = 0; r < 5; ++r) tc::mbar_init(&bars[KV_DRAIN + r], 1);
    *abort_flag = (status != nullptr && (*reinterpret_cast<volatile unsigned*>(status) & kStatusTimeout)) ? 1 : 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(&tm_q);
    tc::tma_prefetch(&tm_do);
    tc::tma_prefetch(&tm_k);
    tc::tma_prefetch(&tm_v);
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const bool issuer = warp < 4 || warp == 8;

  if (issuer) {
    if (lane == 0) {
      volatile int never = 0;
      bool ok = true;
      if (warp == 0) {
        // ------------------------------------------------------------ TMA loader
        constexpr uint32_t kHalfKey = kBK * 128, kHalfRow = kBQ * 128;
        tc::mbar_arrive_expect_tx(&bars[KV_KVFULL], 2 * S::kKeyBytes);
        for (int hf = 0; hf < kHalves; ++hf) {
          tc::tma_load_4d(smem + S::kK + hf * kHalfKey, &tm_k, &bars[KV_KVFULL], 64 * hf, h, kb * kBK, b);
          tc::tma_load_4d(smem + S::kV + hf * kHalfKey, &tm_v, &bars[KV_KVFULL], 64 * hf, h, kb * kBK, b);
        }
        int loaded = 0;
        for (int i = 0; i < n && ok; ++i) {
          const int s = i & 1;
          const int qa = __ldg(qb + i);
          if (i >= 2) ok = tc::wait1(&bars[KV_QFREE + s], ((i >> 1) - 1) & 1, abort_flag);
          if (ok && i >= 2) ok = tc::wait1(&bars[KV_DOFREE + s], ((i >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&bars[KV_QFULL + s], S::kRowBytes);
          tc::mbar_arrive_expect_tx(&bars[KV_DOFULL + s], S::kRowBytes);
          for (int hf = 0; hf < kHalves; ++hf) {
            tc::tma_load_4d(smem + S::kQ + s * S::kRowBytes + hf * kHalfRow, &tm_q, &bars[KV_QFULL + s], 64 * hf, h,
                            qa * kBQ, b);
            tc::tma_load_4d(smem + S::kDO + s * S::kRowBytes + hf * kHalfRow, &tm_do, &bars[KV_DOFULL + s], 64 * hf,
                            h, qa * kBQ, b);
          }
          ++loaded;
        }
        tc::wait1(&bars[KV_KVFULL], 0, &never);
        for (int i = (loaded > 2 ? loaded - 2 : 0); i < loaded; ++i) {
          tc::wait1(&bars[KV_QFULL + (i & 1)], (i >> 1) & 1, &never);
          tc::wait1(&bars[KV_DOFULL + (i & 1)], (i >> 1) & 1, &never);
        }
      } else if (warp == 1 || warp == 2) {
        // ---------------------------------------- S (warp 1) / dP (warp 2) issuer
        const bool is_s = warp == 1;
        constexpr uint32_t idesc = tc::idesc_bf16(128, kBK, false);
        ok = tc::wait1(&bars[KV_KVFULL], 0, abort_flag);
        const unsigned char* b_tile = smem + (is_s ? S::kK : S::kV);
        for (int i = 0; i < n && ok; ++i) {
          const int s = i & 1;
          ok = tc::wait1(&bars[(is_s ? KV_QFULL : KV_DOFULL) + s], (i >> 1) & 1, abort_flag);
          if (ok && i >= 2) ok = tc::wait1(&bars[KV_SFREE + s], ((i >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* a_tile = smem + (is_s ? S::kQ : S::kDO) + s * S::kRowBytes;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int hf = kk / 4, c = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(a_tile + hf * kBQ * 128 + c * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(b_tile + hf * kBK * 128 + c * 32, 16, 1024);
            tc::mma_ss(tmem + (is_s ? kColS : kColDP) + s * kBK, da, db, idesc, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[(is_s ? KV_SFULL : KV_DPFULL) + s]);
        }
      } else {
        // --------------------------- dV (warp 3): dV^T += dO_s^T P; dK (warp 8): dK^T += Q^T dS
        const bool is_v = warp == 3;
        // A = dO_s^T / Q^T (M = d) and B = P / dS (N = 64 keys), both MN-major, K = 128 rows
        constexpr uint32_t idesc = tc::idesc_bf16(128, kBK, true) | (1u << 15);
        const unsigned char* pb = smem + (is_v ? S::kP : S::kDS);
        for (int i = 0; i < n && ok; ++i) {
          const int s = i & 1;
          ok = tc::wait1(&bars[is_v ? KV_PFULL : KV_DSFULL], i & 1, abort_flag);
          if (ok) ok = tc::wait1(&bars[(is_v ? KV_DOFULL : KV_QFULL) + s], (i >> 1) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* a_tile = smem + (is_v ? S::kDO : S::kQ) + s * S::kRowBytes;
#pragma unroll
          for (int kk = 0; kk < kBQ / 16; ++kk) {
            const uint64_t da = tc::smem_desc_sw128(a_tile + kk * 16 * 128, kBQ * 128, 1024);
            const uint64_t db = tc::smem_desc_sw128(pb + kk * 16 * 128, kBQ * 128, 1024);
            tc::mma_ss(tmem + (is_v ? kColDV : kColDK), da, db, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(&bars[is_v ? KV_PFREE : KV_DSFREE]);
          tc::commit(&bars[(is_v ? KV_DOFREE : KV_QFREE) + s]);
        }
      }
      if (warp != 0) {
        const int r = warp == 8 ? 4 : warp;
        tc::commit(&bars[KV_DRAIN + r]);
        tc::wait1(&bars[KV_DRAIN + r], 0, &never);
      }
    }
  } else {
    // -------------------------------------------------------------- compute
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    const int nk = min(kBK, P.L - kb * kBK);  // valid keys of this block
    const float c2 = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
    const float sd = 1.f / sqrtf(static_cast<float>(kD));
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int s = i & 1;
      const int tok = __ldg(qb + i) * kBQ + row;
      const bool row_ok = tok < P.L;
      const size_t rowi = (static_cast<size_t>(b) * P.L + (row_ok ? tok : 0)) * P.H + h;
      const float lse2 = row_ok ? __ldg(lse + rowi) : 0.f;
      const float dsum = row_ok ? __ldg(dd + rowi) : 0.f;
      const int nv = row_ok ? nk : 0;
      ok = tc::wait_warp(&bars[KV_SFULL + s], (i >> 1) & 1, abort_flag);
      if (ok) ok = tc::wait_warp(&bars[KV_DPFULL + s], (i >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::fence_after_sync();
      // P and dS of this row as bf16 pairs, formed 32 keys at a time (S and dP
      // of a half are in registers together) and packed as they are formed
      uint32_t pk_p[kBK / 2], pk_s[kBK / 2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[32], pr[32];
        tc::tmem_ld32p(tmem + lane_base + kColS + s * kBK + 32 * half, sr);
        tc::tmem_ld32p(tmem + lane_base + kColDP + s * kBK + 32 * half, pr);
        tc::tmem_wait_ld();
        if (half == 1) {
          tc::fence_before_sync();
          tc::mbar_arrive(&bars[KV_SFREE + s]);
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int key = 32 * half + c;
          const float p0 = key < nv ? tc::ex2(__uint_as_float(sr[c]) * c2 - lse2) : 0.f;
          const float p1 = key + 1 < nv ? tc::ex2(__uint_as_float(sr[c + 1]) * c2 - lse2) : 0.f;
          pk_p[key / 2] = pack_bf16(p0, p1);
          pk_s[key / 2] = pack_bf16(p0 * (__uint_as_float(pr[c]) - dsum) * sd,
                                    p1 * (__uint_as_float(pr[c + 1]) - dsum) * sd);
        }
      }
      // P of the previous query block has been consumed by its dV MMAs
      if (i > 0) {
        ok = tc::wait_warp(&bars[KV_PFREE], (i - 1) & 1, abort_flag);
        if (!ok) break;
      }
      unsigned char* pbuf = smem + S::kP;
#pragma unroll
      for (int ch = 0; ch < kBK / 8; ++ch)
        *reinterpret_cast<uint4*>(pbuf + sw(row, ch)) =
            make_uint4(pk_p[4 * ch], pk_p[4 * ch + 1], pk_p[4 * ch + 2], pk_p[4 * ch + 3]);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[KV_PFULL]);
      if (i > 0) {
        ok = tc::wait_warp(&bars[KV_DSFREE], (i - 1) & 1, abort_flag);
        if (!ok) break;
      }
      unsigned char* dsb = smem + S::kDS;
#pragma unroll
      for (int ch = 0; ch < kBK / 8; ++ch)
        *reinterpret_cast<uint4*>(dsb + sw(row, ch)) =
            make_uint4(pk_s[4 * ch], pk_s[4 * ch + 1], pk_s[4 * ch + 2], pk_s[4 * ch + 3]);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[KV_DSFULL]);
    }
    // the last dV / dK MMAs have completed: thread = channel c (TMEM lane) adds its
    // 64 keys of dV^T and dK^T into dv and dk (a warp covers 32 consecutive channels)
    if (ok) ok = tc::wait_warp(&bars[KV_PFREE], (n - 1) & 1, abort_flag);
    if (ok) ok = tc::wait_warp(&bars[KV_DSFREE], (n - 1) & 1, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      const int c = row;  // channel
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float* out = part ? dk : dv;
        const uint32_t col = part ? kColDK : kColDV;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[32];
          tc::tmem_ld32(tmem + lane_base + col + 32 * half, r);
          tc::tmem_wait_ld();
          // 16 loads at a time, then their stores: the round trips overlap
          float* base = out + ((static_cast<size_t>(b) * P.L + kb * kBK + 32 * half) * P.H + h) * kD + c;
          const size_t stride = static_cast<size_t>(P.H) * kD;  // one key row
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            float old[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) old[t] = (32 * half + 16 * g + t < nk) ? base[(16 * g + t) * stride] : 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (32 * half + 16 * g + t < nk) base[(16 * g + t) * stride] = old[t] + __uint_as_float(r[16 * g + t]);
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) report_status(status, kStatusTimeout);
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

// [B, L, H, d] bf16 as the 4-D tensor (d, H, L, B); box = 64 channels x `rows` tokens of one head.
bool make_rows_map(CUtensorMap* map, const void* base, const Problem& P, int rows) {
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

}  // namespace

bool backward_tc_supported(const Problem& P) {
  return P.d == kD && P.block_q == kBQ && P.block_k == kBK && !P.causal;
}

cudaError_t launch_backward_attn_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const uint16_t* do_s, const int32_t* block_idx, const int32_t* offs,
                                    const int32_t* list, const float* lse, const float* dd, float* dq, float* dk,
                                    float* dv, unsigned* status, cudaStream_t stream) {
  if (!backward_tc_supported(P)) return cudaErrorInvalidValue;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap mq, mdo, mk, mv, mq2, mdo2;
  if (!make_rows_map(&mq, q, P, kBQ) || !make_rows_map(&mdo, do_s, P, kBQ) || !make_rows_map(&mk, k, P, kBK) ||
      !make_rows_map(&mv, v, P, kBK))
    return cudaErrorInvalidValue;
  mq2 = mq;
  mdo2 = mdo;
  const int smem_dq = DqSmem::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq);
  if (e != cudaSuccess) return e;
  bwd_dq_tc_kernel<<<static_cast<unsigned>(P.B) * P.H * P.n_qblk, kDqThreads, smem_dq, stream>>>(
      mq, mdo, mk, mv, P, block_idx, lse, dd, dq, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int smem_kv = KvSmem::kTotal + 1024;
  e = cudaFuncSetAttribute(bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
  if (e != cudaSuccess) return e;
  bwd_dkv_tc_kernel<<<static_cast<unsigned>(P.B) * P.H * P.n_kblk, kKvThreads, smem_kv, stream>>>(
      mq2, mdo2, mk, mv, P, offs, list, lse, dd, dk, dv, status);
  return cudaGetLastError();
}

}  // namespace sda
