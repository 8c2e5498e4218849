// Low-rank state C = sum_j k~_j v_j^T on the tcgen05 tensor cores (d = 128)
// (SparkDiffusion summary, robotworld.top, section 2.1: features and global
// state equations).
//
// Persistent: one CTA per SM walks work items (batch, head, 2048-token chunk)
// in a fixed round-robin order; each item leaves one r x d partial state.
// Per 128-token tile:
//   warps 0, 6  TMA: the K tiles of one head (128 tokens x d, 128-byte
//               swizzle) into a 2-stage ring freed as soon as U is computed,
//               the V tiles into a 3-stage ring freed by the state MMA;
//   warp 1      one lane issues U = K P_k^T (M=128 tokens, N=r, K=d) into one
//               of two TMEM buffers, and C^T += V^T k~ (M=d, N=r, K=128
//               tokens; A = V read MN-major, B = k~ from shared memory) twice,
//               once with the bf16 head and once with the bf16 tail of k~;
//   warps 2..5  one thread per token: phi and the rank-truncated 3D RoPE on
//               its U row, k~ split into bf16 head + tail and written
//               K-major into shared memory; at the end of an item the same
//               threads (now one per channel) read C^T out of TMEM and write
//               the partial state.
// The accumulator is double-buffered across items, U across tiles. All waits
// are bounded (2 s) and report through the status word.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sda {

namespace {

constexpr int kThreads = 224;  // 7 warps
constexpr int kKStages = 2;
constexpr int kMaxVStages = 3;
// V ring depth: 3 tiles where shared memory allows (r <= 32), else 2
template <int R>
constexpr int v_stages() { return R <= 32 ? 3 : 2; }
constexpr int kTileTok = 128;
constexpr int kChunkTok = 2048;   // tokens per work item (partial state)

template <int R>
struct StateSmem {
  static constexpr int kTileBytes = 2 * kTileTok * 128;        // one d=128 tile: 2 slabs x 128 rows x 128 B
  static constexpr int kKtHalf = 2 * R * 128;                  // one of head/tail: 2 token slabs x R rows x 128 B
  static constexpr int kKtBytes = 2 * kKtHalf;                 // head + tail
  static constexpr int kKRing = 0;                             // kKStages K tiles
  static constexpr int kVRing = kKRing + kKStages * kTileBytes;      // v_stages<R>() V tiles
  static constexpr int kKt = kVRing + v_stages<R>() * kTileBytes;     // 2 buffers
  static constexpr int kPk = kKt + 2 * kKtBytes;               // P_k: 2 d slabs x R rows x 128 B
  static constexpr int kBars = kPk + 2 * R * 128;
  static constexpr int kTotal = kBars + 256;
};

enum {
  SB_KFULL = 0, SB_KEMPTY = 2, SB_VFULL = 4, SB_VEMPTY = 4 + kMaxVStages, SB_UFULL = 4 + 2 * kMaxVStages,
  SB_KTFULL = SB_UFULL + 2, SB_KTEMPTY = SB_KTFULL + 2, SB_CDONE = SB_KTEMPTY + 2, SB_CFREE = SB_CDONE + 2,
  SB_CONSTS = SB_CFREE + 2, SB_DRAIN = SB_CONSTS + 1, SB_N = SB_DRAIN + 1
};

struct Item {
  int bh, chunk, l0, n_tiles;
};

__device__ __forceinline__ Item item_of(const Problem& P, int n_chunks, int it) {
  Item x;
  x.bh = it / n_chunks;
  x.chunk = it % n_chunks;
  x.l0 = x.chunk * kChunkTok;
  const int l1 = min(P.L, x.l0 + kChunkTok);
  x.n_tiles = (l1 - x.l0 + kTileTok - 1) / kTileTok;
  return x;
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
lowrank_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        Problem P, int n_chunks, const float2* __restrict__ tab, const uint16_t* __restrict__ p_k,
                        float* __restrict__ c_part, unsigned* status) {
  constexpr int D = 128;
  using S = StateSmem<R>;
  constexpr int kVStages = v_stages<R>();
  constexpr uint32_t kCols = (4 * R < 32) ? 32 : 4 * R;  // U0, U1, C0, C1 (R columns each)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBars + 8 * SB_N);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBars + 8 * SB_N + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_items = P.B * P.H * n_chunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kVStages; ++s) {
      tc::mbar_init(&bars[SB_VFULL + s], 1);
      tc::mbar_init(&bars[SB_VEMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars[SB_KFULL + s], 1);
      tc::mbar_init(&bars[SB_KEMPTY + s], 1);
      tc::mbar_init(&bars[SB_UFULL + s], 1);
      tc::mbar_init(&bars[SB_KTFULL + s], 128);
      tc::mbar_init(&bars[SB_KTEMPTY + s], 1);
      tc::mbar_init(&bars[SB_CDONE + s], 1);
      tc::mbar_init(&bars[SB_CFREE + s], 128);
    }
    tc::mbar_init(&bars[SB_CONSTS], 128);
    tc::mbar_init(&bars[SB_DRAIN], 1);
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
  // TMEM columns: U buffers at 0 and R, state accumulators at 2R and 3R
  auto colU = [](int ub) { return static_cast<uint32_t>(ub * R); };
  auto colC = [](int cb) { return static_cast<uint32_t>((2 + cb) * R); };

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ producers (K: warp 0, V: warp 6)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int nst = is_k ? kKStages : kVStages;
      uint64_t* full = &bars[is_k ? SB_KFULL : SB_VFULL];
      uint64_t* empty = &bars[is_k ? SB_KEMPTY : SB_VEMPTY];
      unsigned char* ring = smem + (is_k ? S::kKRing : S::kVRing);
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      bool ok = true;
      int gi = 0;  // tiles issued by this CTA
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const Item x = item_of(P, n_chunks, it);
        const int b = x.bh / P.H, h = x.bh % P.H;
        for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
          const int st = gi % nst;
          ok = tc::wait1(&empty[st], ((gi / nst) & 1) ^ 1, abort_flag);
          if (!ok) break;
          unsigned char* dst = ring + st * S::kTileBytes;
          tc::mbar_arrive_expect_tx(&full[st], S::kTileBytes);
          const int l0 = x.l0 + t * kTileTok;
          for (int hf = 0; hf < 2; ++hf) tc::tma_load_4d(dst + hf * kTileTok * 128, map, &full[st], 64 * hf, h, l0, b);
        }
      }
      volatile int never = 0;
      for (int j = gi - nst < 0 ? 0 : gi - nst; j < gi; ++j) tc::wait1(&full[j % nst], (j / nst) & 1, &never);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_u = tc::idesc_bf16(128, R, false);
      // C^T += V^T k~: A = V (M = d contiguous: MN-major), B = k~ (K-major)
      constexpr uint32_t idesc_c = tc::idesc_bf16(128, R, false) | (1u << 15);
      bool ok = tc::wait1(&bars[SB_CONSTS], 0, abort_flag);
      if (ok) tc::fence_after_sync();
      int gi = 0;      // tile counter (stage / U buffer rings)
      int ii = 0;      // item counter (accumulator ring)
      // pending C step: tile (gi - 1) of item (ii_p) when has_prev
      bool has_prev = false;
      int prev_gi = 0, prev_ii = 0;
      bool prev_first = false, prev_last = false;
      auto issue_c = [&](int g, int itn, bool first, bool last) -> bool {
        const int ub = g & 1;
        if (!tc::wait1(&bars[SB_KTFULL + ub], (g >> 1) & 1, abort_flag)) return false;
        if (first && !tc::wait1(&bars[SB_CFREE + (itn & 1)], ((itn >> 1) & 1) ^ 1, abort_flag)) return false;
        tc::fence_after_sync();
        if (!tc::wait1(&bars[SB_VFULL + g % kVStages], (g / kVStages) & 1, abort_flag)) return false;
        tc::fence_after_sync();
        const unsigned char* vt = smem + S::kVRing + (g % kVStages) * S::kTileBytes;
        const unsigned char* kt = smem + S::kKt + ub * S::kKtBytes;
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
#pragma unroll
          for (int kk = 0; kk < kTileTok / 16; ++kk) {
            const uint64_t da = tc::smem_desc_sw128(vt + kk * 16 * 128, kTileTok * 128, 1024);
            const uint64_t db =
                tc::smem_desc_sw128(kt + hl * S::kKtHalf + (kk / 4) * R * 128 + (kk % 4) * 32, 16, 1024);
            tc::mma_ss(tmem + colC(itn & 1), da, db, idesc_c, (first && hl == 0 && kk == 0) ? 0u : 1u);
          }
        }
        tc::commit(&bars[SB_KTEMPTY + ub]);
        tc::commit(&bars[SB_VEMPTY + g % kVStages]);
        if (last) tc::commit(&bars[SB_CDONE + (itn & 1)]);
        return true;
      };
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ii) {
        const Item x = item_of(P, n_chunks, it);
        for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
          const int st = gi % kKStages;
          ok = tc::wait1(&bars[SB_KFULL + st], (gi / kKStages) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          const unsigned char* kt = smem + S::kKRing + st * S::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hf = kk / 4, w = kk % 4;
            const uint64_t da = tc::smem_desc_sw128(kt + hf * kTileTok * 128 + w * 32, 16, 1024);
            const uint64_t db = tc::smem_desc_sw128(smem + S::kPk + hf * R * 128 + w * 32, 16, 1024);
            tc::mma_ss(tmem + colU(gi & 1), da, db, idesc_u, kk > 0 ? 1u : 0u);
          }
          tc::commit(&bars[SB_UFULL + (gi & 1)]);
          tc::commit(&bars[SB_KEMPTY + st]);
          if (has_prev) {
            ok = issue_c(prev_gi, prev_ii, prev_first, prev_last);
            if (!ok) break;
          }
          has_prev = true;
          prev_gi = gi;
          prev_ii = ii;
          prev_first = (t == 0);
          prev_last = (t == x.n_tiles - 1);
        }
      }
      if (ok && has_prev) issue_c(prev_gi, prev_ii, prev_first, prev_last);
      tc::commit(&bars[SB_DRAIN]);
      volatile int never = 0;
      tc::wait1(&bars[SB_DRAIN], 0, &never);
    }
  } else {
    // ------------------------------------------------------------ features + partial-state epilogue
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;  // token of the tile / channel of C^T
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    {
      // P_k (bf16, K-major, 128-byte swizzle) into shared memory for the U MMAs
      const int t = threadIdx.x - 64;
      for (int e = t; e < R * (D / 8); e += 128) {
        const int n = e / (D / 8), c8 = e % (D / 8);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p_k + n * D) + c8);
        *reinterpret_cast<uint4*>(smem + S::kPk + (c8 / 8) * R * 128 + tc::sw128_offset(n, c8 % 8)) = v;
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[SB_CONSTS]);
    }
    bool ok = true;
    int gi = 0, ii = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ii) {
      const Item x = item_of(P, n_chunks, it);
      for (int t = 0; t < x.n_tiles && ok; ++t, ++gi) {
        const int ub = gi & 1;
        ok = tc::wait_warp(&bars[SB_UFULL + ub], (gi >> 1) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        uint32_t ur[R];
#pragma unroll
        for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(tmem + lane_base + colU(ub) + 16 * c, ur + 16 * c);
        tc::tmem_wait_ld();
        const int l = x.l0 + t * kTileTok + row;
        const bool valid = l < P.L;
        const int lc = valid ? l : P.L - 1;
        const int w = lc % P.grid_w;
        const int hh = (lc / P.grid_w) % P.grid_h;
        const int tt = lc / (P.grid_w * P.grid_h);
        const float2* tab_t = tab + tt * P.pairs_t;
        const float2* tab_h = tab + P.grid_t * P.pairs_t + hh * P.pairs_h - P.pairs_t;
        const float2* tab_w = tab + P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + w * P.pairs_w - P.pairs_t - P.pairs_h;
        uint32_t hi2[R / 2], lo2[R / 2];  // packed (k~_{2m}, k~_{2m+1}) head / tail
#pragma unroll
        for (int mm = 0; mm < R / 2; ++mm) {
          const float xx = elu_plus_one(__uint_as_float(ur[2 * mm]));
          const float yy = elu_plus_one(__uint_as_float(ur[2 * mm + 1]));
          const float2* src = mm < P.pairs_t ? tab_t : (mm < P.pairs_t + P.pairs_h ? tab_h : tab_w);
          const float2 cs = __ldg(src + mm);
          const float k0 = valid ? xx * cs.x - yy * cs.y : 0.f;
          const float k1 = valid ? xx * cs.y + yy * cs.x : 0.f;
          float h0, t0, h1, t1;
          split_bf16(k0, h0, t0);
          split_bf16(k1, h1, t1);
          hi2[mm] = pack_bf16(h0, h1);
          lo2[mm] = pack_bf16(t0, t1);
        }
        ok = tc::wait_warp(&bars[SB_KTEMPTY + ub], ((gi >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        // k~ K-major: element (rank n, token `row`) of 2 token slabs x R rows x 128 B
        unsigned char* kt = smem + S::kKt + ub * S::kKtBytes + (row / 64) * R * 128;
        const uint32_t chunk = (row % 64) / 8, within = (row % 8) * 2;
#pragma unroll
        for (int mm = 0; mm < R / 2; ++mm) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int n = 2 * mm + e;
            const uint32_t off = tc::sw128_offset(n, chunk) + within;
            *reinterpret_cast<uint16_t*>(kt + off) = static_cast<uint16_t>(e ? (hi2[mm] >> 16) : (hi2[mm] & 0xffffu));
            *reinterpret_cast<uint16_t*>(kt + S::kKtHalf + off) =
                static_cast<uint16_t>(e ? (lo2[mm] >> 16) : (lo2[mm] & 0xffffu));
          }
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bars[SB_KTFULL + ub]);
      }
      if (!ok) break;
      // partial state of this item: thread `row` holds channel d = row of C^T
      const int cb = ii & 1;
      ok = tc::wait_warp(&bars[SB_CDONE + cb], (ii >> 1) & 1, abort_flag);
      if (!ok) break;
      tc::fence_after_sync();
      uint32_t cr[R];
#pragma unroll
      for (int c = 0; c < R / 16; ++c) tc::tmem_ld16p(tmem + lane_base + colC(cb) + 16 * c, cr + 16 * c);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[SB_CFREE + cb]);
      float* out = c_part + (static_cast<size_t>(x.bh) * n_chunks + x.chunk) * R * D;
#pragma unroll
      for (int m = 0; m < R; ++m) out[m * D + row] = __uint_as_float(cr[m]);
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

template <int R>
cudaError_t run_state_tc(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                         const uint16_t* v, const uint16_t* p_k, float* c_part, unsigned* status,
                         cudaStream_t stream) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, P, kTileTok) || !make_map(&mv, v, P, kTileTok)) return cudaErrorInvalidValue;
  const int smem = StateSmem<R>::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(lowrank_state_tc_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = P.B * P.H * lay.n_split;
  const int grid = n_items < sms ? n_items : sms;
  lowrank_state_tc_kernel<R><<<grid, kThreads, smem, stream>>>(mk, mv, P, lay.n_split, tab, p_k, c_part, status);
  return cudaGetLastError();
}

}  // namespace

int lowrank_state_tc_chunk() { return kChunkTok; }

bool lowrank_state_tc_supported(const Problem& P) { return P.d == 128; }

cudaError_t launch_lowrank_state_tc(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                                    const uint16_t* v, const uint16_t* p_k, float* c_part, unsigned* status,
                                    cudaStream_t stream) {
  if (P.rank == 16) return run_state_tc<16>(P, lay, tab, k, v, p_k, c_part, status, stream);
  if (P.rank == 32) return run_state_tc<32>(P, lay, tab, k, v, p_k, c_part, status, stream);
  if (P.rank == 64) return run_state_tc<64>(P, lay, tab, k, v, p_k, c_part, status, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sda
