// Host side of the C ABI declared in include/sda.h: argument checks, workspace
// layout, launch order. No device memory is allocated here.

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/sda.h"
#include "common.cuh"
#include "kernels.h"

using sda::Layout;
using sda::Problem;

namespace {

thread_local std::string g_detail;

int32_t fail(int32_t code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int32_t fail(int32_t code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_detail = buf;
  return code;
}

constexpr size_t kAlign = 256;
constexpr int kStateCtasPerSm = 2;  // resident state CTAs per SM: the chunking aims at one full wave
constexpr int kSmCount = 148;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

}  // namespace

namespace sda {

int32_t set_error(int32_t code, const char* msg) { return fail(code, "%s", msg); }

int32_t make_problem(const sda_params* p, Problem* P) {
  if (p == nullptr) return fail(SDA_ERR_NULLPTR, "params is NULL");
  if (p->B < 1 || p->L < 1 || p->H < 1) return fail(SDA_ERR_SHAPE, "B, L, H must be >= 1");
  if (p->d != 64 && p->d != 128) return fail(SDA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", p->d);
  if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1 ||
      static_cast<int64_t>(p->grid_t) * p->grid_h * p->grid_w != p->L)
    return fail(SDA_ERR_SHAPE, "L (%d) != grid_t*grid_h*grid_w (%d*%d*%d)", p->L, p->grid_t, p->grid_h, p->grid_w);
  if (p->block_q != 64 && p->block_q != 128)
    return fail(SDA_ERR_UNSUPPORTED, "block_q must be 64 or 128 (got %d)", p->block_q);
  if (p->block_k != 64) return fail(SDA_ERR_UNSUPPORTED, "block_k must be 64 (got %d)", p->block_k);
  if (!(p->sparsity >= 0.0 && p->sparsity < 1.0)) return fail(SDA_ERR_SHAPE, "sparsity must lie in [0, 1)");
  if (p->rank != 16 && p->rank != 32 && p->rank != 64)
    return fail(SDA_ERR_UNSUPPORTED, "rank must be 16, 32 or 64 (got %d)", p->rank);
  if (p->pairs_t < 0 || p->pairs_h < 0 || p->pairs_w < 0 || p->pairs_t + p->pairs_h + p->pairs_w != p->rank / 2)
    return fail(SDA_ERR_SHAPE, "pairs_t + pairs_h + pairs_w must equal rank / 2");
  if (!(p->rope_base > 0.0) || !std::isfinite(p->rope_base)) return fail(SDA_ERR_SHAPE, "rope_base must be > 0");
  if (!(p->rms_eps >= 0.0) || !std::isfinite(p->rms_eps)) return fail(SDA_ERR_SHAPE, "rms_eps must be >= 0");
  if (p->gate_per_head != 0 && p->gate_per_head != 1) return fail(SDA_ERR_SHAPE, "gate_per_head must be 0 or 1");
  if (p->causal_frames < 0 || p->causal_frames > p->grid_t ||
      (p->causal_frames > 0 && p->grid_t % p->causal_frames != 0))
    return fail(SDA_ERR_SHAPE, "causal_frames (%d) must be 0 or divide grid_t (%d)", p->causal_frames, p->grid_t);
  const int64_t elems = static_cast<int64_t>(p->B) * p->L * p->H * p->d;
  if (elems >= (int64_t(1) << 40)) return fail(SDA_ERR_UNSUPPORTED, "tensor too large");
  if (static_cast<int64_t>(p->B) * p->H * ((p->L + 63) / 64) >= (int64_t(1) << 31))
    return fail(SDA_ERR_UNSUPPORTED, "too many blocks for one launch");

  std::memset(P, 0, sizeof(*P));
  P->B = p->B;
  P->L = p->L;
  P->H = p->H;
  P->d = p->d;
  P->grid_t = p->grid_t;
  P->grid_h = p->grid_h;
  P->grid_w = p->grid_w;
  P->block_q = p->block_q;
  P->block_k = p->block_k;
  P->n_qblk = (p->L + p->block_q - 1) / p->block_q;
  P->n_kblk = (p->L + p->block_k - 1) / p->block_k;
  P->keep_ratio = 1.0 - p->sparsity;
  const double kf = std::ceil(P->keep_ratio * P->n_kblk - 1e-6);
  int keep = static_cast<int>(kf);
  if (keep < 1) keep = 1;
  if (keep > P->n_kblk) keep = P->n_kblk;
  P->keep = keep;
  P->rank = p->rank;
  P->pairs_t = p->pairs_t;
  P->pairs_h = p->pairs_h;
  P->pairs_w = p->pairs_w;
  P->rms_eps = static_cast<float>(p->rms_eps);
  P->rope_base = p->rope_base;
  P->gate_per_head = p->gate_per_head;
  const int counts[3] = {p->pairs_t, p->pairs_h, p->pairs_w};
  int m = 0;
  for (int ax = 0; ax < 3; ++ax)
    for (int mu = 0; mu < counts[ax]; ++mu) P->theta[m++] = std::pow(p->rope_base, -static_cast<double>(mu) / counts[ax]);

  P->causal = p->causal_frames > 0 ? 1 : 0;
  if (P->causal) {
    P->chunk_tokens = p->causal_frames * p->grid_h * p->grid_w;
    P->n_chunks = p->grid_t / p->causal_frames;
    P->nq_chunk = (P->chunk_tokens + p->block_q - 1) / p->block_q;
    P->n_qblk = P->n_chunks * P->nq_chunk;
    P->n_kcols = P->n_kblk + P->n_chunks;
  } else {
    P->chunk_tokens = p->L;
    P->n_chunks = 1;
    P->nq_chunk = P->n_qblk;
    P->n_kcols = P->n_kblk;
  }
  if (P->n_kblk > sda::kMaxKeyBlocks)
    return fail(SDA_ERR_UNSUPPORTED, "N_kblk = %d exceeds the selector's limit of %d key blocks", P->n_kblk,
                sda::kMaxKeyBlocks);
  return SDA_OK;
}

Layout make_layout(const Problem& P) {
  Layout y{};
  const size_t BH = static_cast<size_t>(P.B) * P.H;
  int n_split, split_len, n_sub;
  if (sda::lowrank_state_tc_supported(P)) {
    // persistent tcgen05 state kernel: pieces of 256..2048 tokens, one partial state each,
    // tiling every causal chunk (the whole sequence without a window) on its own
    split_len = sda::lowrank_state_tc_chunk(P);
    n_sub = (P.chunk_tokens + split_len - 1) / split_len;
    n_split = P.n_chunks * n_sub;
  } else {
    // warp-MMA state kernel: every causal chunk (the whole sequence without a
    // window) in n_sub pieces of split_len tokens, about one wave of CTAs in all
    const int max_sub = (P.chunk_tokens + 63) / 64;
    n_sub = static_cast<int>((kStateCtasPerSm * kSmCount) / (BH * P.n_chunks));
    if (n_sub < 1) n_sub = 1;
    if (n_sub > max_sub) n_sub = max_sub;
    split_len = (P.chunk_tokens + n_sub - 1) / n_sub;
    split_len = (split_len + 63) / 64 * 64;
    n_sub = (P.chunk_tokens + split_len - 1) / split_len;
    n_split = P.n_chunks * n_sub;
  }
  y.n_split = n_split;
  y.split_len = split_len;
  y.n_sub = n_sub;
  const size_t NC = static_cast<size_t>(P.n_chunks);
  size_t off = 0;
  y.status = off;       off = align_up(off + 4);
  y.q_mean = off;       off = align_up(off + BH * P.n_qblk * P.d * 4);   // bf16 head + tail
  y.k_mean = off;       off = align_up(off + BH * P.n_kcols * P.d * 4);
  y.scores = off;       off = align_up(off + sda::score_workspace_bytes(P));
  y.block_idx = off;    off = align_up(off + BH * P.n_qblk * P.keep * 4);
  y.c_part = off;       off = align_up(off + BH * n_split * P.rank * P.d * 4);
  y.c_state = off;      off = align_up(off + BH * NC * P.rank * P.d * 4);
  y.ct_f32 = off;       off = align_up(off + BH * NC * P.rank * P.d * 4);
  y.ct_hi = off;        off = align_up(off + BH * NC * P.rank * P.d * 2);
  y.ct_lo = off;        off = align_up(off + BH * NC * P.rank * P.d * 2);
  y.rope_tab = off;     off = align_up(off + static_cast<size_t>(sda::rope_table_entries(P)) * 8);
  y.total = off;
  return y;
}

}  // namespace sda

namespace {

using sda::make_layout;
using sda::make_problem;

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(SDA_ERR_NULLPTR, "%s is NULL", name);
  if (!aligned16(p)) return fail(SDA_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return SDA_OK;
}

int32_t check_ws(const Layout& y, void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(SDA_ERR_NULLPTR, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return fail(SDA_ERR_ALIGN, "workspace is not 256-byte aligned");
  if (ws_bytes < y.total) return fail(SDA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, y.total);
  return SDA_OK;
}

// The kernels are built for sm_100a only: check the current device once per device.
int32_t check_device() {
  static std::mutex mu;
  static int checked[64] = {0};  // 0 unknown, 1 ok, -1 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(SDA_ERR_DEVICE, "no CUDA device");
  if (dev < 0 || dev >= 64) return fail(SDA_ERR_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    checked[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (checked[dev] != 1) return fail(SDA_ERR_DEVICE, "device %d is not sm_100 (the kernels are built for sm_100a)", dev);
  return SDA_OK;
}

int32_t launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(SDA_ERR_LAUNCH, "%s: %s", what, cudaGetErrorString(e));
  return SDA_OK;
}

#define SDA_TRY(x)            \
  do {                        \
    int32_t rc_ = (x);        \
    if (rc_ != SDA_OK) return rc_; \
  } while (0)

int32_t common_checks(const sda_params* p, Problem* P, Layout* y, void* ws, size_t ws_bytes) {
  SDA_TRY(make_problem(p, P));
  *y = make_layout(*P);
  SDA_TRY(check_ws(*y, ws, ws_bytes));
  SDA_TRY(check_device());
  return SDA_OK;
}

}  // namespace

extern "C" {

int32_t sda_keep_count(const sda_params* p) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  return P.keep;
}

int32_t sda_query_blocks(const sda_params* p) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  return P.n_qblk;
}

size_t sda_workspace_size(const sda_params* p) {
  Problem P;
  if (make_problem(p, &P) != SDA_OK) return 0;
  return make_layout(P).total;
}

int32_t sda_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr) return fail(SDA_ERR_NULLPTR, "workspace is NULL");
  if (ws_bytes < 4) return fail(SDA_ERR_WORKSPACE, "workspace too small");
  SDA_TRY(check_device());
  return launched(cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)), "cudaMemsetAsync");
}

int32_t sda_read_status(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr) return fail(SDA_ERR_NULLPTR, "workspace is NULL");
  if (ws_bytes < 4) return fail(SDA_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(SDA_ERR_DEVICE, "reading the status word: %s", cudaGetErrorString(e));
  if (word == 0) return SDA_OK;
  e = cudaMemsetAsync(ws, 0, 4, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (word & sda::kStatusTimeout) return fail(SDA_ERR_TIMEOUT, "a bounded in-kernel wait ran out (status 0x%x)", word);
  return fail(SDA_ERR_SHAPE, "a block index outside its candidates ([0, N_kblk), or [0, n_c) in causal chunk c) "
                             "was skipped (status 0x%x)", word);
}

int32_t sda_block_select(const sda_params* p, const uint16_t* q, const uint16_t* k, int32_t* block_idx, void* ws,
                         size_t ws_bytes, void* stream) {
  Problem P;
  Layout y;
  SDA_TRY(common_checks(p, &P, &y, ws, ws_bytes));
  SDA_TRY(check_ptr(q, "q"));
  SDA_TRY(check_ptr(k, "k"));
  SDA_TRY(check_ptr(block_idx, "block_idx"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launched(sda::launch_block_select(P, q, k, at<uint16_t>(ws, y.q_mean), at<uint16_t>(ws, y.k_mean),
                                          at<float>(ws, y.scores), block_idx, at<unsigned>(ws, y.status),
                                          /*pool_k=*/true, s),
                  "block select");
}

int32_t sda_sparse_attn_fwd(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const int32_t* block_idx, uint16_t* o_s, void* ws, size_t ws_bytes, void* stream) {
  Problem P;
  Layout y;
  SDA_TRY(common_checks(p, &P, &y, ws, ws_bytes));
  SDA_TRY(check_ptr(q, "q"));
  SDA_TRY(check_ptr(k, "k"));
  SDA_TRY(check_ptr(v, "v"));
  SDA_TRY(check_ptr(block_idx, "block_idx"));
  SDA_TRY(check_ptr(o_s, "o_s"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launched(sda::launch_sparse_attn_tc(P, q, k, v, block_idx, o_s, at<unsigned>(ws, y.status), s),
                  "sparse attention");
}

int32_t sda_lowrank_fwd(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* p_q, const uint16_t* p_k, uint16_t* o_lr, float* c_out, void* ws,
                        size_t ws_bytes, void* stream) {
  Problem P;
  Layout y;
  SDA_TRY(common_checks(p, &P, &y, ws, ws_bytes));
  SDA_TRY(check_ptr(q, "q"));
  SDA_TRY(check_ptr(k, "k"));
  SDA_TRY(check_ptr(v, "v"));
  SDA_TRY(check_ptr(p_q, "p_q"));
  SDA_TRY(check_ptr(p_k, "p_k"));
  SDA_TRY(check_ptr(o_lr, "o_lr"));
  if (c_out != nullptr) SDA_TRY(check_ptr(c_out, "c_out"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float2* tab = at<float2>(ws, y.rope_tab);
  SDA_TRY(launched(sda::launch_rope_table(P, tab, s), "rope table"));
  SDA_TRY(launched(sda::launch_lowrank_state(P, y, tab, k, v, p_k, at<float>(ws, y.c_part), at<float>(ws, y.c_state),
                                             c_out, nullptr, at<uint16_t>(ws, y.ct_hi), at<uint16_t>(ws, y.ct_lo),
                                             at<unsigned>(ws, y.status), true, nullptr, s),
                   "low-rank state"));
  return launched(sda::launch_lowrank_readout(P, tab, q, p_q, at<uint16_t>(ws, y.ct_hi), at<uint16_t>(ws, y.ct_lo),
                                              o_lr, at<unsigned>(ws, y.status), true, s),
                  "low-rank readout");
}

size_t sda_backward_workspace_size(const sda_params* p) {
  Problem P;
  if (make_problem(p, &P) != SDA_OK) return 0;
  return sda::backward_workspace_bytes(P, make_layout(P));
}

int32_t sda_backward(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const uint16_t* p_q, const uint16_t* p_k, const float* g, const int32_t* block_idx,
                     const uint16_t* d_o, float* dq, float* dk, float* dv, float* dp_q, float* dp_k, float* dg,
                     void* ws, size_t ws_bytes, void* stream) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  const Layout y = make_layout(P);
  const size_t need = sda::backward_workspace_bytes(P, y);
  if (ws == nullptr) return fail(SDA_ERR_NULLPTR, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return fail(SDA_ERR_ALIGN, "workspace is not 256-byte aligned");
  if (ws_bytes < need) return fail(SDA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  const void* ins[] = {q, k, v, p_q, p_k, g, block_idx, d_o};
  const char* in_names[] = {"q", "k", "v", "p_q", "p_k", "g", "block_idx", "d_o"};
  for (int i = 0; i < 8; ++i) SDA_TRY(check_ptr(ins[i], in_names[i]));
  void* outs[] = {dq, dk, dv, dp_q, dp_k, dg};
  const char* out_names[] = {"dq", "dk", "dv", "dp_q", "dp_k", "dg"};
  for (int i = 0; i < 6; ++i) SDA_TRY(check_ptr(outs[i], out_names[i]));
  SDA_TRY(check_device());
  return launched(sda::launch_backward(P, y, ws, q, k, v, p_q, p_k, g, block_idx, d_o, dq, dk, dv, dp_q, dp_k, dg,
                                       static_cast<cudaStream_t>(stream)),
                  "backward");
}

int32_t sda_gate_fuse(const sda_params* p, const uint16_t* o_s, const uint16_t* o_lr, const float* g, uint16_t* o,
                      void* stream) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  SDA_TRY(check_device());
  SDA_TRY(check_ptr(o_s, "o_s"));
  SDA_TRY(check_ptr(o_lr, "o_lr"));
  SDA_TRY(check_ptr(g, "g"));
  SDA_TRY(check_ptr(o, "o"));
  return launched(sda::launch_gate_fuse(P, o_s, o_lr, g, o, static_cast<cudaStream_t>(stream)), "gate");
}

int32_t sda_qk_prologue(const sda_params* p, const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* w_q,
                        const uint16_t* w_k, uint16_t* q_norm, uint16_t* k_norm, uint16_t* q_rot, uint16_t* k_rot,
                        void* stream) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  if (!sda::qk_prologue_supported(P))
    return fail(SDA_ERR_UNSUPPORTED, "the full-d rotation table (%d x (d/8) + %d x (3d/16) + %d x (3d/16)) "
                "exceeds 8192 entries", P.grid_t, P.grid_h, P.grid_w);
  SDA_TRY(check_device());
  const void* ptrs[] = {q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot};
  const char* names[] = {"q_raw", "k_raw", "w_q", "w_k", "q_norm", "k_norm", "q_rot", "k_rot"};
  for (int i = 0; i < 8; ++i) SDA_TRY(check_ptr(ptrs[i], names[i]));
  return launched(sda::launch_qk_prologue(P, q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot,
                                          static_cast<cudaStream_t>(stream)),
                  "q/k prologue");
}

int32_t sda_quant_fp8(const sda_params* p, const uint16_t* x, uint8_t* x_q, float* scale, void* stream) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  if (P.H * P.d > sda::quant_fp8_max_row())
    return fail(SDA_ERR_UNSUPPORTED, "H*d = %d exceeds %d channels per token", P.H * P.d, sda::quant_fp8_max_row());
  SDA_TRY(check_device());
  SDA_TRY(check_ptr(x, "x"));
  SDA_TRY(check_ptr(x_q, "x_q"));
  SDA_TRY(check_ptr(scale, "scale"));
  return launched(sda::launch_quant_fp8(P, x, x_q, scale, static_cast<cudaStream_t>(stream)), "fp8 quantisation");
}

static int32_t forward_impl(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const uint16_t* p_q, const uint16_t* p_k, const float* g, uint16_t* o,
                            int32_t* block_idx_out, void* ws, size_t ws_bytes, void* const* events, void* stream) {
  Problem P;
  Layout y;
  SDA_TRY(common_checks(p, &P, &y, ws, ws_bytes));
  SDA_TRY(check_ptr(q, "q"));
  SDA_TRY(check_ptr(k, "k"));
  SDA_TRY(check_ptr(v, "v"));
  SDA_TRY(check_ptr(p_q, "p_q"));
  SDA_TRY(check_ptr(p_k, "p_k"));
  SDA_TRY(check_ptr(g, "g"));
  SDA_TRY(check_ptr(o, "o"));
  if (block_idx_out != nullptr) SDA_TRY(check_ptr(block_idx_out, "block_idx_out"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> int32_t {
    if (events == nullptr) return SDA_OK;
    return launched(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s), "cudaEventRecord");
  };
  int32_t* idx = block_idx_out ? block_idx_out : at<int32_t>(ws, y.block_idx);
  float2* tab = at<float2>(ws, y.rope_tab);
  // The state pass streams all of K anyway; where it can, it also leaves the key
  // block means in the workspace and the selector pools only Q.
  const bool state_pools_k = sda::lowrank_state_tc_pools_k(P);
  uint16_t* k_mean = at<uint16_t>(ws, y.k_mean);
  SDA_TRY(mark(0));
  SDA_TRY(launched(sda::launch_rope_table(P, tab, s), "rope table"));
  SDA_TRY(launched(sda::launch_lowrank_state(P, y, tab, k, v, p_k, at<float>(ws, y.c_part), at<float>(ws, y.c_state),
                                             nullptr, at<float>(ws, y.ct_f32), at<uint16_t>(ws, y.ct_hi),
                                             at<uint16_t>(ws, y.ct_lo), at<unsigned>(ws, y.status), true,
                                             state_pools_k ? k_mean : nullptr, s),
                   "low-rank state"));
  SDA_TRY(mark(1));
  SDA_TRY(launched(sda::launch_block_select(P, q, k, at<uint16_t>(ws, y.q_mean), k_mean, at<float>(ws, y.scores),
                                            idx, at<unsigned>(ws, y.status), !state_pools_k, s),
                   "block select"));
  SDA_TRY(mark(2));
  // the low-rank readout and the gate run inside the tcgen05 attention epilogue
  SDA_TRY(mark(3));
  SDA_TRY(launched(sda::launch_sparse_attn_tc_fused(P, q, k, v, idx, p_q, at<uint16_t>(ws, y.ct_hi),
                                                    at<uint16_t>(ws, y.ct_lo), tab, g, o, at<unsigned>(ws, y.status), s),
                   "fused sparse attention"));
  return mark(4);
}

int32_t sda_forward(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const uint16_t* p_q, const uint16_t* p_k, const float* g, uint16_t* o, int32_t* block_idx_out,
                    void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(p, q, k, v, p_q, p_k, g, o, block_idx_out, ws, ws_bytes, nullptr, stream);
}

int32_t sda_forward_profiled(const sda_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const uint16_t* p_q, const uint16_t* p_k, const float* g, uint16_t* o,
                             int32_t* block_idx_out, void* ws, size_t ws_bytes, void* const* events, void* stream) {
  if (events == nullptr) return fail(SDA_ERR_NULLPTR, "events is NULL");
  for (int i = 0; i < 5; ++i)
    if (events[i] == nullptr) return fail(SDA_ERR_NULLPTR, "events[%d] is NULL", i);
  return forward_impl(p, q, k, v, p_q, p_k, g, o, block_idx_out, ws, ws_bytes, events, stream);
}

size_t sda_forward_host_buffer_size(const sda_params* p) {
  Problem P;
  if (make_problem(p, &P) != SDA_OK) return 0;
  const Layout y = make_layout(P);
  const size_t tensor = static_cast<size_t>(P.B) * P.L * P.H * P.d * 2;
  const size_t proj = static_cast<size_t>(P.rank) * P.d * 2;
  const size_t gate = static_cast<size_t>(P.B) * P.L * (P.gate_per_head ? P.H : 1) * 4;
  return y.total + 4 * align_up(tensor) + 2 * align_up(proj) + align_up(gate);
}

int32_t sda_forward_host(const sda_params* p, const uint16_t* q_host, const uint16_t* k_host, const uint16_t* v_host,
                         const uint16_t* p_q_host, const uint16_t* p_k_host, const float* g_host, uint16_t* o_host,
                         void* dev_buf, size_t dev_buf_bytes, void* stream) {
  Problem P;
  SDA_TRY(make_problem(p, &P));
  if (!q_host || !k_host || !v_host || !p_q_host || !p_k_host || !g_host || !o_host)
    return fail(SDA_ERR_NULLPTR, "a host buffer is NULL");
  const size_t need = sda_forward_host_buffer_size(p);
  if (dev_buf == nullptr) return fail(SDA_ERR_NULLPTR, "dev_buf is NULL");
  if (dev_buf_bytes < need) return fail(SDA_ERR_WORKSPACE, "dev_buf has %zu bytes, needs %zu", dev_buf_bytes, need);
  const Layout y = make_layout(P);
  const size_t tensor = static_cast<size_t>(P.B) * P.L * P.H * P.d * 2;
  const size_t proj = static_cast<size_t>(P.rank) * P.d * 2;
  const size_t gate = static_cast<size_t>(P.B) * P.L * (P.gate_per_head ? P.H : 1) * 4;
  unsigned char* base = static_cast<unsigned char*>(dev_buf);
  size_t off = y.total;
  auto take = [&](size_t n) {
    unsigned char* r = base + off;
    off += align_up(n);
    return r;
  };
  uint16_t* dq = reinterpret_cast<uint16_t*>(take(tensor));
  uint16_t* dk = reinterpret_cast<uint16_t*>(take(tensor));
  uint16_t* dv = reinterpret_cast<uint16_t*>(take(tensor));
  uint16_t* dpq = reinterpret_cast<uint16_t*>(take(proj));
  uint16_t* dpk = reinterpret_cast<uint16_t*>(take(proj));
  float* dg = reinterpret_cast<float*>(take(gate));
  uint16_t* dout = reinterpret_cast<uint16_t*>(take(tensor));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SDA_TRY(check_device());
  const struct {
    void* dst;
    const void* src;
    size_t n;
  } copies[] = {{dq, q_host, tensor}, {dk, k_host, tensor}, {dv, v_host, tensor},
                {dpq, p_q_host, proj}, {dpk, p_k_host, proj}, {dg, g_host, gate}};
  for (const auto& c : copies) {
    cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return fail(SDA_ERR_DEVICE, "host-to-device copy: %s", cudaGetErrorString(e));
  }
  SDA_TRY(sda_forward(p, dq, dk, dv, dpq, dpk, dg, dout, nullptr, dev_buf, y.total, stream));
  cudaError_t e = cudaMemcpyAsync(o_host, dout, tensor, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(SDA_ERR_DEVICE, "device-to-host copy: %s", cudaGetErrorString(e));
  return sda_read_status(dev_buf, y.total, stream);
}

uint64_t sda_set_attention_wait_limit_ns(uint64_t limit_ns) { return sda::set_attention_wait_limit(limit_ns); }

const char* sda_error_string(int32_t code) {
  switch (code) {
    case SDA_OK: return "ok";
    case SDA_ERR_NULLPTR: return "null pointer";
    case SDA_ERR_ALIGN: return "misaligned pointer";
    case SDA_ERR_SHAPE: return "inconsistent shape or parameter";
    case SDA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SDA_ERR_WORKSPACE: return "workspace too small";
    case SDA_ERR_LAUNCH: return "kernel launch failed";
    case SDA_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    case SDA_ERR_DEVICE: return "CUDA device / runtime error";
    default: return "unknown error";
  }
}

const char* sda_last_error_detail(void) { return g_detail.c_str(); }

const char* sda_version(void) { return "sda 0.1.0 sm_100a"; }

}  // extern "C"
