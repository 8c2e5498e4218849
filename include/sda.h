/*
 * sda.h -- C ABI of the B200 (sm_100a) compensated sparse attention forward.
 *
 * The operation (SparkDiffusion summary on robotworld.top, section 2.1,
 * "compensated sparse attention"):
 *
 *   O_i  = O_s,i + g_i * r_i * O_lr,i
 *   O_s  = A_M(Q, K, V)       block-sparse softmax(Q K^T / sqrt(d)) V over the
 *                             key blocks kept for the query's block
 *   O_lr = RMSNorm(q~_i^T C)  C = sum_j k~_j v_j^T
 *   q~_i = R_r(p_i) phi(P_q q_i),  k~_j = R_r(p_j) phi(P_k k_j)
 *   r_i  = RMS over d of O_s,i
 *
 * Readings where the pages leave a step open: blocks are contiguous runs of
 * raster-ordered tokens; the selector mean-pools Q and K per block, scores
 * pooled pairs by their dot product and keeps the best
 * k = ceil((1 - s) * N_kblk - 1e-6) (clamped to [1, N_kblk]) key blocks per
 * (batch, head, query block), ties to the lower index; phi = elu + 1; R_r
 * turns adjacent pairs (2m, 2m+1), the first pairs_t by the token's t
 * coordinate, the next pairs_h by h, the rest by w, pair mu of an axis with
 * n pairs at frequency rope_base^(-mu / n); RMSNorm has no weight.
 *
 * Conventions shared by every call:
 *  - Tensors are dense, row-major, in device memory owned by the caller.
 *    Q, K, V, O, O_s, O_lr: [B, L, H, d] bf16 (raw bits in uint16_t), the
 *    Wan attention layout. P_q, P_k: [r, d] bf16. g: [B, L] fp32 (or
 *    [B, L, H] when gate_per_head). block_idx: [B, H, N_qblk, k] int32,
 *    kept key-block indices of each query block in ascending order.
 *  - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and never synchronises the host. Every argument
 *    is checked on the host before any launch; on error nothing is launched
 *    and a negative SDA_ERR_* code is returned. sda_last_error_detail()
 *    gives a one-line reason for the last error of the calling thread.
 *  - Outputs are fully overwritten; inputs are never written; outputs must
 *    not alias inputs.
 *  - Sizes the kernels take: d in {64, 128}; block_k = 64; block_q in
 *    {64, 128}; r in {16, 32, 64}; N_kblk = ceil(L / 64) <= 2048 (L up to
 *    131,072 tokens). Anything else returns SDA_ERR_UNSUPPORTED.
 *  - The library holds no device memory between calls, except the fixed
 *    scratch array of sda_lowrank_fwd_static (below). Scratch space comes
 *    from the caller's workspace of sda_workspace_size() bytes, which must
 *    be passed through sda_workspace_init() once after allocation (it clears
 *    the sticky status word that kernels with bounded waits report into).
 */
#ifndef SDA_H
#define SDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define SDA_OK 0
#define SDA_ERR_NULLPTR (-1)     /* a required pointer is NULL */
#define SDA_ERR_ALIGN (-2)       /* a pointer is not 16-byte (workspace: 256-byte) aligned */
#define SDA_ERR_SHAPE (-3)       /* inconsistent sizes (e.g. L != grid_t*grid_h*grid_w) */
#define SDA_ERR_UNSUPPORTED (-4) /* valid but outside what the kernels implement */
#define SDA_ERR_WORKSPACE (-5)   /* workspace smaller than sda_workspace_size() */
#define SDA_ERR_LAUNCH (-6)      /* a kernel launch failed (cudaGetLastError) */
#define SDA_ERR_TIMEOUT (-7)     /* a bounded in-kernel wait ran out (see sda_read_status) */
#define SDA_ERR_DEVICE (-8)      /* no usable sm_100 device / CUDA runtime error */

/* Problem description. */
typedef struct sda_params {
  int32_t B, L, H, d;              /* batch, tokens, heads, head dim (d in {64, 128}) */
  int32_t grid_t, grid_h, grid_w;  /* token grid; L == grid_t * grid_h * grid_w, raster order */
  int32_t block_q, block_k;        /* query / key block sizes: block_q in {64, 128}, block_k == 64 */
  double sparsity;                 /* s in [0, 1) */
  int32_t rank;                    /* r in {16, 32, 64} */
  int32_t pairs_t, pairs_h, pairs_w; /* RoPE pairs per axis, sum == r / 2 */
  double rope_base;                /* > 1, e.g. 10000 */
  double rms_eps;                  /* RMSNorm eps of the low-rank readout, e.g. 1e-6 */
  int32_t gate_per_head;           /* 0: g is [B, L]; 1: g is [B, L, H] */
  int32_t causal_frames;           /* 0: bidirectional; F > 0: causal window of F-frame chunks
                                      (F must divide grid_t), see below */
} sda_params;

/* Causal-window variant (robotworld summary, section 4: the compensated sparse
 * attention restricted to a causal window for autoregressive generation).
 * With causal_frames = F > 0 the tokens form chunks of F whole latent frames,
 * Tc = F * grid_h * grid_w tokens each, and the queries of chunk c see exactly
 * the keys of chunks 0..c (tokens below hi_c = (c + 1) * Tc). Every step is
 * the bidirectional one applied to that prefix:
 *  - query blocks tile each chunk on its own (N_qblk = (grid_t / F) *
 *    ceil(Tc / block_q); sda_query_blocks() gives it), the last block of a
 *    chunk may be partial;
 *  - the selector scores the key blocks of [0, hi_c), the last one pooled
 *    over its visible tokens only, and keeps k_c = clamp(ceil((1 - s) n_c -
 *    1e-6), 1, n_c) of the n_c = ceil(hi_c / block_k) candidates; a row of
 *    block_idx holds those k_c indices in ascending order followed by -1 up
 *    to the width k = sda_keep_count() of the last chunk;
 *  - the sparse attention of a chunk-c query attends to the kept blocks' keys
 *    below hi_c; the kernels read only the first k_c entries of each row, and
 *    an entry at or past n_c counts as a bad index;
 *  - the low-rank state of chunk c is the prefix C_c = sum over j < hi_c of
 *    k~_j v_j^T, and a chunk-c query reads out C_c.
 * No output of chunk c depends on a token of a later chunk. */

/* Number of query blocks N_qblk of the block map: ceil(L / block_q), or
 * (grid_t / F) * ceil(Tc / block_q) with a causal window. Negative SDA_ERR_*
 * on bad parameters. */
int32_t sda_query_blocks(const sda_params* p);

/* Number of kept key blocks per query block (the row width of block_idx),
 * k = clamp(ceil((1 - s) * N_kblk - 1e-6), 1, N_kblk): the sparse branch keeps
 * a 1 - s fraction of query-key blocks (robotworld summary, section 1; the
 * README's `topk` argument is this keep ratio). Negative SDA_ERR_* on bad
 * parameters. */
int32_t sda_keep_count(const sda_params* p);

/* Bytes of device workspace that every call below may use (0 on bad params). */
size_t sda_workspace_size(const sda_params* p);

/* Zero the workspace's status word (call once after allocating it). */
int32_t sda_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read the sticky status word of `ws` and clear it.
 * Returns SDA_OK; SDA_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last read; SDA_ERR_SHAPE if the sparse attention met a block index outside
 * [0, N_kblk) (with a causal window: outside the [0, n_c) candidates of the
 * query block's chunk) and skipped it. The affected outputs are then undefined. */
int32_t sda_read_status(void* ws, size_t ws_bytes, void* stream);

/* Block selector (robotworld summary, section 2.1: A_M keeps a 1 - s
 * fraction of query-key blocks chosen by block-level scoring / top-k).
 * Mean-pools q over each query block and k over each key block (partial last
 * blocks over their valid tokens, fp32 accumulation in a fixed order), scores
 * every pooled pair by its dot product and writes the top-k key blocks of
 * every (batch, head, query block) to block_idx in ascending order, ties to
 * the lower index. The means are kept as a bf16 head plus a bf16 tail and a
 * score is the fp32-accumulated sum of three bf16 products (head.head +
 * head.tail + tail.head): about 16 significant bits, so two scores closer
 * than ~2^-16 of the row's largest may be ranked either way; the map equals
 * the exact top-k whenever the k-th and (k+1)-th scores of a row differ by
 * more than that. q, k: [B, L, H, d] bf16. block_idx: [B, H, N_qblk, k].
 * With a causal window: per chunk over its prefix, rows padded with -1 (see
 * the causal-window paragraph above). */
int32_t sda_block_select(const sda_params* p, const uint16_t* q, const uint16_t* k,
                         int32_t* block_idx, void* ws, size_t ws_bytes, void* stream);

/* Block-sparse attention A_M (robotworld summary, section 2.1, dense formula
 * restricted to the kept blocks): for every query row i of block a,
 * O_s,i = softmax_j(q_i . k_j / sqrt(d)) v_j over the valid keys j of the key
 * blocks block_idx[b, h, a, :], renormalised over that set. bf16 inputs,
 * fp32 accumulation and softmax, bf16 output o_s: [B, L, H, d]. block_idx
 * entries must lie in [0, N_kblk) (checked on the device: bad entries are
 * skipped and reported through the status word). With a causal window a
 * chunk-c block reads the first k_c entries of its row, which must lie in
 * [0, n_c), and attends to keys below hi_c only. */
int32_t sda_sparse_attn_fwd(const sda_params* p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const int32_t* block_idx, uint16_t* o_s,
                            void* ws, size_t ws_bytes, void* stream);

/* Low-rank branch (robotworld summary, section 2.1, feature / state /
 * readout equations): C[b, h] = sum over all valid tokens j of k~_j v_j^T
 * (r x d, fp32, split over token chunks and reduced in a fixed order), then
 * o_lr_i = RMSNorm(q~_i^T C) over d (eps = rms_eps). p_q, p_k: [r, d] bf16,
 * shared by all heads. o_lr: [B, L, H, d] bf16. c_out: [B, H, r, d] fp32, or
 * NULL to skip writing C. With a causal window: c_out is [B, H, n_chunks, r, d]
 * (the prefix states C_c) and a chunk-c row reads out C_c. */
int32_t sda_lowrank_fwd(const sda_params* p, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                        uint16_t* o_lr, float* c_out, void* ws, size_t ws_bytes, void* stream);

/* sda_lowrank_fwd for callers that cannot allocate device memory. The paper
 * has no counterpart: this is a deployment variant of the low-rank branch.
 * Some callers cannot provide the workspace sda_lowrank_fwd needs -- e.g. a
 * host application whose memory planner owns every device allocation and
 * gives a plug-in only its inputs and outputs, or a path on which cudaMalloc's
 * implicit device synchronisation is not allowed. This entry point computes
 * the same C and O_lr with the warp-MMA state and readout kernels (those
 * report no bounded-wait status, which needs a workspace word), so it matches
 * sda_lowrank_fwd to rounding, not bit for bit. Its scratch lives in a fixed
 * 32 MiB file-scope device array that every GPU loading the library holds
 * until the process exits; it calls no cudaMalloc, cudaFree or allocating
 * routine. Arguments are those of sda_lowrank_fwd without the workspace.
 * Problems whose scratch exceeds 32 MiB are rejected with
 * SDA_ERR_UNSUPPORTED; the scratch is B*H*n_split*r*d*4 (chunk partials of C)
 * + B*H*n_chunks*r*d*8 (C and the bf16 head/tail of C^T) bytes plus the RoPE
 * table, each region rounded up to 256 bytes, with n_split ~ 296 / (B*H)
 * token pieces per head (at least one per causal chunk) and n_chunks = 1
 * without a causal window. The first call in each CUDA context (normally:
 * the first call on each device, with that device current) looks up the
 * array's device address with cudaGetSymbolAddress and caches it under the
 * context; make that first call before any stream capture. All calls share
 * the one array: calls that overlap on the GPU (other streams, other
 * threads) race, so the caller must serialise them. The array keeps the last
 * call's contents; every region is fully written before it is read within a
 * call, so nothing in it needs to start at zero. */
int32_t sda_lowrank_fwd_static(const sda_params* p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                               uint16_t* o_lr, float* c_out, void* stream);

/* Backward of the forward (training backpropagates through both branches:
 * the sparse warm-up trains the low-rank projections and the gate and needs
 * a backward of the sparse attention; H3 portability report, sections
 * 2.1-2.2). Gradients of sum(O * d_o) for O = sda_forward's output, with the
 * block map held fixed (it carries no gradient):
 *   dq, dk, dv: [B, L, H, d] fp32 (both branches summed); dp_q, dp_k: [r, d]
 *   fp32 (summed over every batch, token and head); dg: like g, fp32.
 * Inputs: those of sda_forward, block_idx the map sda_forward returned (rows
 * ascending, as the selector writes them), d_o: [B, L, H, d] bf16. The call
 * recomputes C, O_s and O_lr with the forward kernels, then runs the chain
 * rule in reverse (gate; RMSNorm, readout and query features; state and key
 * features; softmax of the kept blocks) with fp32 accumulation, every sum in
 * a fixed order (bit-identical reruns). At d = 128 the sparse branch's
 * products run on the tensor cores with bf16 operands (P and dS rounded to
 * bf16; 128-row query blocks, no window) and, at r = 16 or 32, the low-rank
 * products with every fp32 operand split into a bf16 head and tail (about
 * fp32 accuracy); other shapes run those steps in fp32 on the CUDA cores. ws: sda_backward_workspace_size() bytes, passed
 * through sda_workspace_init once. A map entry outside [0, N_kblk) is skipped
 * and reported through the status word (with a causal window the -1 padding
 * of a row is skipped silently). With a causal window (causal_frames > 0) the
 * gradients are those of the causal forward: a row of chunk c reads the prefix
 * state C_c, so key j receives the sum of dC_c over the chunks c that hold it
 * in their prefix, and the sparse branch sees the keys below hi_c only. */
size_t sda_backward_workspace_size(const sda_params* p);
int32_t sda_backward(const sda_params* p, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                     const float* g, const int32_t* block_idx, const uint16_t* d_o, float* dq,
                     float* dk, float* dv, float* dp_q, float* dp_k, float* dg, void* ws,
                     size_t ws_bytes, void* stream);

/* Gate fusion (robotworld summary, section 2.1, last equation):
 * o_i = o_s,i + g_i * r_i * o_lr,i with r_i = sqrt(mean_c o_s,i,c^2) from the
 * bf16 o_s given here. o_s, o_lr, o: [B, L, H, d] bf16; g: [B, L] or
 * [B, L, H] fp32. */
int32_t sda_gate_fuse(const sda_params* p, const uint16_t* o_s, const uint16_t* o_lr,
                      const float* g, uint16_t* o, void* stream);

/* Prologue of the path (SparkDiffusion summary, robotworld.top, section 2.1:
 * the low-rank branch reuses the backbone's normalised q/k; the sparse
 * branch attends with the rotated ones): per (token, head) row of q_raw and
 * of k_raw, x_norm = x / sqrt(mean_c x_c^2 + rms_eps) * w and x_rot = the
 * full-d 3D RoPE of x_norm (all d/2 adjacent pairs; (d/8, 3d/16, 3d/16)
 * pairs to the (t, h, w) axes, pair mu of an axis with n pairs turning by
 * coordinate * rope_base^(-mu / n)), both rounded to bf16 from the same fp32
 * x_norm. q_raw, k_raw, q_norm, k_norm, q_rot, k_rot: [B, L, H, d] bf16;
 * w_q, w_k: [H, d] bf16 (the backbone's learned norm weights). q_rot/k_rot
 * feed sda_block_select and sda_sparse_attn_fwd, q_norm/k_norm feed
 * sda_lowrank_fwd. Outputs may not alias inputs. A rotation table of more
 * than 8192 (axis coordinate, pair) entries -> SDA_ERR_UNSUPPORTED. */
int32_t sda_qk_prologue(const sda_params* p, const uint16_t* q_raw, const uint16_t* k_raw,
                        const uint16_t* w_q, const uint16_t* w_k, uint16_t* q_norm,
                        uint16_t* k_norm, uint16_t* q_rot, uint16_t* k_rot, void* stream);

/* Per-token FP8 E4M3 quantisation of an activation tensor, scale and cast in
 * one pass (SparkDiffusion summary, robotworld.top, section 2.3: activations
 * of the linear projections in E4M3 with a per-token scale chosen at run
 * time), e.g. of the forward's output o before the output projection.
 * x: [B, L, H, d] bf16; a token's row is its H*d channels. x_q: [B, L, H, d]
 * E4M3 bytes; scale: [B, L] fp32, x ~ E4M3-decode(x_q) * scale. Per row:
 * amax = max |x|, x_q = E4M3(x * (448 / amax)) with round-to-nearest-even,
 * saturated at +-448, sign of zero kept; scale = amax / 448 (both quotients
 * and the product in IEEE fp32); a row of zeros gets scale 1 and zero codes.
 * Only B, L, H, d of p are used (p must still be valid). H*d > 16384 ->
 * SDA_ERR_UNSUPPORTED. x_q may not alias x. */
int32_t sda_quant_fp8(const sda_params* p, const uint16_t* x, uint8_t* x_q, float* scale,
                      void* stream);

/* The whole forward: low-rank state, selector, low-rank readout, then the
 * sparse attention with the gate applied in its epilogue, where r_i comes
 * from the unrounded fp32 sparse output. With d = 128 and r <= 32 the state
 * pass also forms the key block means, so the selector pools only Q; the
 * block map is the same either way. o: [B, L, H, d] bf16. block_idx_out:
 * [B, H, N_qblk, k] int32 or NULL (the map then stays in the workspace). */
int32_t sda_forward(const sda_params* p, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                    const float* g, uint16_t* o, int32_t* block_idx_out, void* ws,
                    size_t ws_bytes, void* stream);

/* sda_forward with stage timing: records events[0..4] (cudaEvent_t handles
 * created by the caller) on `stream` before the low-rank state, before the
 * selector, before the low-rank readout, before the sparse attention and
 * after it. Same launches and results as sda_forward. */
int32_t sda_forward_profiled(const sda_params* p, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, const uint16_t* p_q, const uint16_t* p_k,
                             const float* g, uint16_t* o, int32_t* block_idx_out, void* ws,
                             size_t ws_bytes, void* const* events, void* stream);

/* Device bytes sda_forward_host needs in `dev_buf`: staging for q, k, v,
 * p_q, p_k, g and o plus the workspace. */
size_t sda_forward_host_buffer_size(const sda_params* p);

/* sda_forward from and to HOST memory: copies q, k, v, p_q, p_k, g into
 * dev_buf with one cudaMemcpyAsync each, runs sda_forward there and copies o
 * back into the host buffer, then synchronises `stream`. Host buffers should
 * be pinned (page-locked) for the copies to run at full speed. dev_buf
 * (device, 256-byte aligned, sda_forward_host_buffer_size bytes) must have
 * been passed through sda_workspace_init at offset 0 once; the call checks
 * the status word before returning. */
int32_t sda_forward_host(const sda_params* p, const uint16_t* q_host, const uint16_t* k_host,
                         const uint16_t* v_host, const uint16_t* p_q_host,
                         const uint16_t* p_k_host, const float* g_host, uint16_t* o_host,
                         void* dev_buf, size_t dev_buf_bytes, void* stream);

/* Failure-detection diagnostic: sets the time limit, in nanoseconds, of the
 * waits on pipeline progress (TMA tiles landed, MMAs done, softmax tiles
 * handed over) in the tcgen05 sparse attention kernel of sda_sparse_attn_fwd
 * and sda_forward, for every launch made after the call, from any thread;
 * returns the previous limit. The default is 2e9 (2 s, far beyond any
 * legitimate wait). 0 makes a wait give up unless its phase is already
 * complete at the first, non-blocking test, so a launch then reliably takes
 * the failure path: the CTA records SDA_ERR_TIMEOUT in the workspace status
 * word (sda_read_status), waits -- with the 2 s limit -- for its own TMA
 * loads and MMAs in flight, frees its tensor memory and exits; its outputs are
 * undefined, and later launches skip their work until the status is read.
 * Meant for tests of that path; not for production use. */
uint64_t sda_set_attention_wait_limit_ns(uint64_t limit_ns);

/* Static description of an error code. */
const char* sda_error_string(int32_t code);

/* One-line reason for the last error returned to the calling thread. */
const char* sda_last_error_detail(void);

/* Library version, e.g. "sda 0.1.0 sm_100a". */
const char* sda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDA_H */
