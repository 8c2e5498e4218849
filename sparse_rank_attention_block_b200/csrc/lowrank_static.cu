// Low-rank branch for callers that cannot allocate device memory.
//
// sda_lowrank_fwd needs a caller-provided workspace. Some callers cannot get
// one at call time: a host application whose memory planner owns every device
// allocation and hands a plug-in only its inputs and outputs, or a code path
// where cudaMalloc's implicit device synchronisation is not allowed. For them
// sda_lowrank_fwd_static runs the same kernels with their scratch (chunk
// partials of C, C, C^T head/tail, RoPE table) in a fixed file-scope device
// array instead. Every GPU that loads this library holds that array until the
// process exits.

#include <cuda.h>

#include <mutex>

#include "../../include/sda.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Host code must not use this name as a device address: it is a host-side
// stand-in. The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_lowrank_scratch[kStaticScratchBytes];

// A __device__ array's address belongs to a CUDA context, not to a device: a
// host that makes its own driver-API context current, or that recreates the
// primary context (cudaDeviceReset), sees the array at another address. The
// address is therefore looked up once per context, keyed by the context's
// process-unique ID (cuCtxGetId; IDs are never reused, so a context created
// at the address of a destroyed one still gets its own entry).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct CtxEntry {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kMaxContexts = 64;
std::mutex g_mu;
CtxEntry g_entries[kMaxContexts];
int g_n_entries = 0;

template <class Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Device address of the scratch array in the current context. The first call
// in a context (with cudart's primary context: the first call on a device)
// looks it up with cudaGetSymbolAddress and caches it under the context ID.
int32_t scratch_address(unsigned char** out) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_current == nullptr || get_id == nullptr)
    return sda::set_error(SDA_ERR_DEVICE, "the driver lacks cuCtxGetCurrent / cuCtxGetId");
  auto current_id = [&](unsigned long long* id) {
    CUcontext ctx = nullptr;
    return get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr && get_id(ctx, id) == CUDA_SUCCESS;
  };
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = 0;
  const bool have_ctx = current_id(&id);
  if (have_ctx)
    for (int i = 0; i < g_n_entries; ++i)
      if (g_entries[i].ctx_id == id) {
        *out = static_cast<unsigned char*>(g_entries[i].addr);
        return SDA_OK;
      }
  // Set-up in this context. With no context current yet (a thread that has
  // made no CUDA call), the runtime makes the current device's primary
  // context current here, and that is the context the launches then use.
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_lowrank_scratch);
  if (e != cudaSuccess || p == nullptr)
    return sda::set_error(SDA_ERR_DEVICE, "cudaGetSymbolAddress of the static scratch failed");
  if (!have_ctx && !current_id(&id))
    return sda::set_error(SDA_ERR_DEVICE, "no current CUDA context after looking up the static scratch");
  // keep the most recent contexts: a full table drops its oldest entry
  if (g_n_entries == kMaxContexts) {
    for (int i = 1; i < kMaxContexts; ++i) g_entries[i - 1] = g_entries[i];
    --g_n_entries;
  }
  g_entries[g_n_entries++] = CtxEntry{id, p};
  *out = static_cast<unsigned char*>(p);
  return SDA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int32_t sda_lowrank_fwd_static(const sda_params* p, const uint16_t* q, const uint16_t* k,
                                          const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                                          uint16_t* o_lr, float* c_out, void* stream) {
  sda::Problem P;
  const int32_t rc = sda::make_problem(p, &P);
  if (rc != SDA_OK) return rc;
  const uint16_t* ins[] = {q, k, v, p_q, p_k};
  for (const uint16_t* x : ins)
    if (x == nullptr) return sda::set_error(SDA_ERR_NULLPTR, "an input pointer is NULL");
  if (o_lr == nullptr) return sda::set_error(SDA_ERR_NULLPTR, "o_lr is NULL");
  for (const uint16_t* x : ins)
    if (!aligned16(x)) return sda::set_error(SDA_ERR_ALIGN, "an input pointer is not 16-byte aligned");
  if (!aligned16(o_lr) || (c_out != nullptr && !aligned16(c_out)))
    return sda::set_error(SDA_ERR_ALIGN, "an output pointer is not 16-byte aligned");

  // Same token chunks as sda_lowrank_fwd; the partial states come from the
  // warp-MMA state kernel here (no status word to report a bounded-wait
  // time-out through), so the two agree to rounding, not bit for bit.
  const sda::Layout lay = sda::make_layout(P);
  const size_t BH = static_cast<size_t>(P.B) * P.H;
  const size_t BHC = BH * P.n_chunks;  // one state per causal chunk (one without a window)
  const size_t rd = static_cast<size_t>(P.rank) * P.d;
  size_t off = 0;
  const size_t o_part = off;  off = align_up(off + BH * lay.n_split * rd * 4);
  const size_t o_state = off; off = align_up(off + BHC * rd * 4);
  const size_t o_hi = off;    off = align_up(off + BHC * rd * 2);
  const size_t o_lo = off;    off = align_up(off + BHC * rd * 2);
  const size_t o_tab = off;   off = align_up(off + static_cast<size_t>(sda::rope_table_entries(P)) * 8);
  if (off > kStaticScratchBytes)
    return sda::set_error(SDA_ERR_UNSUPPORTED,
                          "problem needs more than the 32 MiB static scratch of sda_lowrank_fwd_static "
                          "(B*H*n_split*r*d*4 + B*H*n_chunks*r*d*8 bytes); use sda_lowrank_fwd with a workspace");

  int dev = -1;
  cudaGetDevice(&dev);
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return sda::set_error(SDA_ERR_DEVICE, "device is not sm_100 (the kernels are built for sm_100a)");

  unsigned char* base = nullptr;
  const int32_t src = scratch_address(&base);
  if (src != SDA_OK) return src;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float2* tab = reinterpret_cast<float2*>(base + o_tab);
  uint16_t* ct_hi = reinterpret_cast<uint16_t*>(base + o_hi);
  uint16_t* ct_lo = reinterpret_cast<uint16_t*>(base + o_lo);
  // Every scratch region is fully written before it is read inside one call:
  // nothing has to start at zero.
  cudaError_t e = sda::launch_rope_table(P, tab, s);
  if (e == cudaSuccess)
    e = sda::launch_lowrank_state(P, lay, tab, k, v, p_k, reinterpret_cast<float*>(base + o_part),
                                  reinterpret_cast<float*>(base + o_state), c_out, nullptr, ct_hi, ct_lo,
                                  nullptr, /*use_tc=*/false, /*k_mean=*/nullptr, s);
  if (e == cudaSuccess) e = sda::launch_lowrank_readout(P, tab, q, p_q, ct_hi, ct_lo, o_lr, nullptr, /*use_tc=*/false, s);
  if (e != cudaSuccess) return sda::set_error(SDA_ERR_LAUNCH, cudaGetErrorString(e));
  return SDA_OK;
}
