// Internal launcher declarations of the sda kernels (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sda.h"
#include "common.cuh"

namespace sda {

// sda_api.cu: argument checks and workspace layout shared by the entry points.
int32_t make_problem(const sda_params* p, Problem* P);
Layout make_layout(const Problem& P);
int32_t set_error(int32_t code, const char* msg);  // records the detail, returns code

// select.cu
// Longest key-block row the selector takes (its top-k keeps a row in registers).
constexpr int kMaxKeyBlocks = 2048;
size_t score_workspace_bytes(const Problem& P);  // fp32 scores, rows padded to 256 key blocks
// q_mean / k_mean: [B, H, N, 2d] bf16 rows (head then tail, natural channel order);
// scores: score_workspace_bytes; status: workspace status word (bounded-wait
// time-outs are reported there)
// pool_k false: k_mean already holds the key block means (the state kernel made them)
cudaError_t launch_block_select(const Problem& P, const uint16_t* q, const uint16_t* k, uint16_t* q_mean,
                                uint16_t* k_mean, float* scores, int32_t* block_idx, unsigned* status,
                                bool pool_k, cudaStream_t stream);

// lowrank.cu
size_t lowrank_state_smem_bytes(const Problem& P);
size_t lowrank_readout_smem_bytes(const Problem& P);
cudaError_t launch_rope_table(const Problem& P, float2* tab, cudaStream_t stream);
// Writes C (fp32 [B,H,r,d]), optionally c_out (same), C^T fp32 ([B,H,d,r], may be
// NULL) and C^T as bf16 head / tail ([B,H,d,r] each). With use_tc and d = 128 the
// partial states come from the persistent tcgen05 kernel (lowrank_tc.cu), which
// reports bounded-wait time-outs through `status`; otherwise from the warp-MMA kernel.
// k_mean (may be NULL): with use_tc and lowrank_state_tc_pools_k(P), the state
// kernel also writes the key block means the selector scores with.
cudaError_t launch_lowrank_state(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                                 const uint16_t* v, const uint16_t* p_k, float* c_part, float* c_state,
                                 float* c_out, float* ct_f32, uint16_t* ct_hi, uint16_t* ct_lo,
                                 unsigned* status, bool use_tc, uint16_t* k_mean, cudaStream_t stream);

// lowrank_tc.cu
int lowrank_state_tc_chunk(const Problem& P);    // tokens per partial state (256..2048)
bool lowrank_state_tc_supported(const Problem& P);
bool lowrank_state_tc_pools_k(const Problem& P);  // the tcgen05 state kernel can produce the key block means
cudaError_t launch_lowrank_state_tc(const Problem& P, const Layout& lay, const float2* tab, const uint16_t* k,
                                    uint16_t* k_mean,
                                    const uint16_t* v, const uint16_t* p_k, float* c_part, unsigned* status,
                                    cudaStream_t stream);
// use_tc: the tcgen05 readout where lowrank_readout_tc_supported(P) (status: the
// word its bounded waits report to), else the warp-MMA kernel.
cudaError_t launch_lowrank_readout(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                                   const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr, unsigned* status,
                                   bool use_tc, cudaStream_t stream);
bool lowrank_readout_tc_supported(const Problem& P);  // d = 128, r in {16, 32}
cudaError_t launch_lowrank_readout_tc(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                                      const uint16_t* ct_hi, const uint16_t* ct_lo, uint16_t* o_lr,
                                      unsigned* status, cudaStream_t stream);

// gate.cu
cudaError_t launch_gate_fuse(const Problem& P, const uint16_t* o_s, const uint16_t* o_lr, const float* g,
                             uint16_t* o, cudaStream_t stream);

// prologue.cu: backbone RMSNorm (weight [H, d]) and full-d 3D RoPE of q and k
bool qk_prologue_supported(const Problem& P);  // the cos/sin table fits in shared memory
cudaError_t launch_qk_prologue(const Problem& P, const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* w_q,
                               const uint16_t* w_k, uint16_t* q_norm, uint16_t* k_norm, uint16_t* q_rot,
                               uint16_t* k_rot, cudaStream_t stream);

// quant.cu: per-token E4M3 codes and scales of a [B, L, H, d] bf16 tensor
int quant_fp8_max_row();  // largest H*d one warp holds
cudaError_t launch_quant_fp8(const Problem& P, const uint16_t* x, uint8_t* xq, float* scale, cudaStream_t stream);

// sparse_attn_tc.cu: the block-sparse attention on tcgen05 (64-key blocks; a
// CTA takes a 128-row query block or two adjacent 64-row ones). The plain form
// writes O_s; the fused form also computes the low-rank readout from C^T as
// bf16 head / tail ([B,H,d,r] each) and applies the gate, writing O.
bool sparse_attn_tc_supported(const Problem& P);
// Limit of the tcgen05 attention kernel's waits on pipeline progress for the
// launches that follow (default 2 s; 0: give up unless already complete).
// Returns the previous limit.
uint64_t set_attention_wait_limit(uint64_t limit_ns);
// lse (optional, [B, L, H] fp32): log2 of each row's softmax denominator with
// the scaled reference folded in, so that P = 2^(s * log2(e) / sqrt(d) - lse).
cudaError_t launch_sparse_attn_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const int32_t* block_idx, uint16_t* o_s, unsigned* status, cudaStream_t stream,
                                  float* lse = nullptr);
cudaError_t launch_sparse_attn_tc_fused(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                        const int32_t* block_idx, const uint16_t* p_q, const uint16_t* ct_hi,
                                        const uint16_t* ct_lo, const float2* rope_tab, const float* g, uint16_t* o,
                                        unsigned* status, cudaStream_t stream);

// backward_tc.cu: the sparse branch's dq, dk, dv on the tensor cores (d = 128,
// 128-row query blocks, no causal window). do_s: bf16 [B, L, H, d]; offs/list:
// the transposed map; lse: log2-sum-exp2 per row (launch_sparse_attn_tc);
// dd = dO_s . O_s per row. Adds into dq, dk, dv.
bool backward_tc_supported(const Problem& P);
// backward_lr_tc.cu: the low-rank branch of the backward on tcgen05 (d = 128, r = 16 or 32).
// CTAs per (batch, causal chunk, head) group; the partials of dC ([group][cta][r*d]) and of
// dP_q / dP_k ([group * cta][r*d]) are summed in CTA order by outer_reduce_kernel.
bool lr_tc_supported(const Problem& P);
int lr_tc_ctas_per_group(const Problem& P);
cudaError_t launch_lr_q_tc(const Problem& P, const float2* tab, const uint16_t* q, const uint16_t* p_q,
                           const float* c_state, const float* dy, float* dq, float* part_c, float* part_p,
                           unsigned* status, cudaStream_t s);
cudaError_t launch_lr_k_tc(const Problem& P, const float2* tab, const uint16_t* k, const uint16_t* v,
                           const uint16_t* p_k, const float* gsum, float* dk, float* dv, float* part_p,
                           unsigned* status, cudaStream_t s);
cudaError_t launch_backward_attn_tc(const Problem& P, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const uint16_t* do_s, const int32_t* block_idx, const int32_t* offs,
                                    const int32_t* list, const float* lse, const float* dd, float* dq, float* dk,
                                    float* dv, unsigned* status, cudaStream_t stream);

// backward.cu: gradients of sum(O * dO) after a forward recompute; its
// scratch follows the forward's workspace regions.
size_t backward_workspace_bytes(const Problem& P, const Layout& fy);
cudaError_t launch_backward(const Problem& P, const Layout& fy, void* ws, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k, const float* g,
                            const int32_t* block_idx, const uint16_t* d_o, float* dq, float* dk, float* dv,
                            float* dp_q, float* dp_k, float* dg, cudaStream_t stream);

}  // namespace sda
