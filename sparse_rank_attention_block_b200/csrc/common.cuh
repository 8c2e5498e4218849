// Shared device/host definitions of the sda library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace sda {

constexpr int kMaxRank = 64;
constexpr int kMaxPairs = kMaxRank / 2;

// Status bits the kernels OR into the workspace's status word.
constexpr unsigned kStatusTimeout = 1u;      // a bounded wait ran out
constexpr unsigned kStatusBadIndex = 2u;     // a block index outside [0, N_kblk)

// Everything a kernel needs to know about the problem, passed by value.
struct Problem {
  int B, L, H, d;
  int grid_t, grid_h, grid_w;
  int block_q, block_k;
  int n_qblk, n_kblk, keep;
  int rank, pairs_t, pairs_h, pairs_w;
  float rms_eps;
  int gate_per_head;
  double rope_base;         // base of the rotation frequencies
  double theta[kMaxPairs];  // angular frequency of every rotation pair
  // Causal window (chunks of whole latent frames; the queries of chunk c see
  // the keys of chunks 0..c). Without a window the sequence is one chunk:
  // chunk_tokens = L, n_chunks = 1, nq_chunk = n_qblk, n_kcols = n_kblk.
  int causal;               // 0 / 1
  int chunk_tokens;         // tokens per chunk (L = n_chunks * chunk_tokens)
  int n_chunks;
  int nq_chunk;             // query blocks per chunk (n_qblk = n_chunks * nq_chunk)
  int n_kcols;              // pooled key rows: N_kblk, plus one edge row per chunk when causal
  double keep_ratio;        // 1 - s
};

// ---------------------------------------------------------------------------
// causal-window geometry (every helper reduces to the bidirectional case
// when the whole sequence is one chunk)
// ---------------------------------------------------------------------------

// One past the last token the queries of chunk c may see.
__host__ __device__ inline int chunk_end(const Problem& P, int c) { return (c + 1) * P.chunk_tokens; }
// Query blocks tile each chunk on their own: block a covers [start, end).
__host__ __device__ inline int qblk_chunk(const Problem& P, int a) { return a / P.nq_chunk; }
__host__ __device__ inline int qblk_start(const Problem& P, int a) {
  return (a / P.nq_chunk) * P.chunk_tokens + (a % P.nq_chunk) * P.block_q;
}
__host__ __device__ inline int qblk_end(const Problem& P, int a) {
  const int e = qblk_start(P, a) + P.block_q, c = chunk_end(P, a / P.nq_chunk);
  return e < c ? e : c;
}
// Candidate key blocks of chunk c: those holding a token below chunk_end(c).
__host__ __device__ inline int chunk_cands(const Problem& P, int c) {
  return (chunk_end(P, c) + P.block_k - 1) / P.block_k;
}
// Key blocks kept out of n candidates: clamp(ceil((1 - s) n - 1e-6), 1, n),
// in the same IEEE double operations as the host (no contraction).
__device__ inline int keep_of(const Problem& P, int n) {
  if (!P.causal) return P.keep;
  const double x = __dsub_rn(__dmul_rn(P.keep_ratio, static_cast<double>(n)), 1e-6);
  int k = static_cast<int>(ceil(x));
  if (k < 1) k = 1;
  if (k > n) k = n;
  return k;
}

// Workspace regions (byte offsets from the workspace base).
struct Layout {
  size_t status;      // unsigned status word (+ padding)
  size_t q_mean;      // [B, H, N_qblk, 2d] bf16: mean head then tail
  size_t k_mean;      // [B, H, n_kcols, 2d] bf16
  size_t scores;      // [B, H, N_qblk, n_kcols padded to 256] fp32 pooled scores
  size_t block_idx;   // [B, H, N_qblk, k] int32
  size_t c_part;      // [B, H, n_split, r, d] fp32
  size_t c_state;     // [B, H, n_chunks, r, d] fp32 (prefix states when causal)
  size_t ct_f32;      // [B, H, n_chunks, d, r] fp32 C^T
  size_t ct_hi;       // [B, H, n_chunks, d, r] bf16 head of C^T
  size_t ct_lo;       // [B, H, n_chunks, d, r] bf16 tail of C^T
  size_t rope_tab;    // float2 cos/sin table
  size_t total;
  int n_split;        // token pieces of the state build (n_chunks * n_sub)
  int split_len;      // tokens per piece (multiple of 64)
  int n_sub;          // pieces per causal chunk (the whole sequence when there is no window)
};

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Split x into a bf16 head and a bf16 tail: x ~= head + tail to ~16 mantissa bits.
__device__ __forceinline__ void split_bf16(float x, float& head, float& tail) {
  head = __bfloat162float(__float2bfloat16_rn(x));
  tail = x - head;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// cp.async 16 bytes global -> shared; src_bytes 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void report_status(unsigned* status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

// phi(u) = elu(u) + 1.
__device__ __forceinline__ float elu_plus_one(float u) { return u > 0.f ? u + 1.f : expf(u); }

// RoPE tables: cos / sin of coordinate * theta for every (axis value, pair of
// that axis), computed in double and rounded to fp32. Layout in `tab`
// (float2 = {cos, sin}): t-block [grid_t][pairs_t], then h-block
// [grid_h][pairs_h], then w-block [grid_w][pairs_w].
__host__ __device__ inline int rope_table_entries(const Problem& P) {
  return P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + P.grid_w * P.pairs_w;
}

__device__ inline void build_rope_table(const Problem& P, float2* tab) {
  const int nt = P.grid_t * P.pairs_t, nh = P.grid_h * P.pairs_h, nw = P.grid_w * P.pairs_w;
  for (int e = threadIdx.x; e < nt + nh + nw; e += blockDim.x) {
    int coord, pair;
    if (e < nt) {
      coord = e / P.pairs_t;
      pair = e % P.pairs_t;
    } else if (e < nt + nh) {
      coord = (e - nt) / P.pairs_h;
      pair = P.pairs_t + (e - nt) % P.pairs_h;
    } else {
      coord = (e - nt - nh) / P.pairs_w;
      pair = P.pairs_t + P.pairs_h + (e - nt - nh) % P.pairs_w;
    }
    double s, c;
    sincos(static_cast<double>(coord) * P.theta[pair], &s, &c);
    tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// cos/sin of pair m for the token at raster index l.
__device__ __forceinline__ float2 rope_lookup(const Problem& P, const float2* tab, int l, int m) {
  const int w = l % P.grid_w;
  const int h = (l / P.grid_w) % P.grid_h;
  const int t = l / (P.grid_w * P.grid_h);
  if (m < P.pairs_t) return tab[t * P.pairs_t + m];
  if (m < P.pairs_t + P.pairs_h) return tab[P.grid_t * P.pairs_t + h * P.pairs_h + (m - P.pairs_t)];
  return tab[P.grid_t * P.pairs_t + P.grid_h * P.pairs_h + w * P.pairs_w + (m - P.pairs_t - P.pairs_h)];
}

}  // namespace sda
