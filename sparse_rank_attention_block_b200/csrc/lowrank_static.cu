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

#include <mutex>

#include "../../include/sda.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kAlign = 256;

// Host code must not use this name as a device address: it is a host-side
// stand-in. The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_lowrank_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
int32_t scratch_address(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return sda::set_error(SDA_ERR_DEVICE, "no usable CUDA device for the static scratch");
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_lowrank_scratch);
    if (e != cudaSuccess || p == nullptr)
      return sda::set_error(SDA_ERR_DEVICE, "cudaGetSymbolAddress of the static scratch failed");
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
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
