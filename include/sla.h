/*
 * sla.h - C ABI of the Sparse-Linear Attention (SLA / SLA2) forward on B200.
 *
 * Sources (cited by page title and section):
 *   [SLA]  "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
 *          Sparse-Linear Attention": §2 Q2 (algorithm steps 1-4), §3 Fig. 4
 *          (forward flowchart), §4 (notation table, Eq. 3-4, Eq. 6, check 5),
 *          §7 (code cross-reference).
 *   [SLA2] "SLA2: Sparse-Linear Attention with Learnable Routing and QAT":
 *          §3 SLA2 Design, §4 Learnable Router, §5 Quantization-aware Training.
 *
 * Conventions shared by every call
 *   - Tensors Q, K, V, O are bf16 [B, H, N, d] with the head dimension
 *     contiguous; strides of the B, H and N dimensions are given in elements
 *     in sla_params_t (they must be multiples of 8 elements; base pointers
 *     16-byte aligned).
 *   - The caller owns and allocates every device buffer, including the
 *     workspace (size from sla_workspace_size).  The library allocates nothing
 *     on the device and never synchronises the stream, except
 *     sla_get_device_status which reads back the device error word.
 *   - All compute calls are asynchronous on `stream`.  Arguments are validated
 *     on the host before any launch; a rejected call launches nothing.
 *   - Kernels never trap.  A wait that cannot complete within one second, or
 *     a LUT entry out of range, is recorded in the workspace's device error
 *     word and the kernel returns; sla_get_device_status reports it.
 *   - T_q = ceil(N / b_q), T_kv = ceil(N / b_kv).  The last block may be
 *     partial; its pooled mean is over its real tokens.
 *   - Supported: d in {64, 128}, b_q = b_kv = 64, N <= 262144, B*H <= 65535.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sla_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, bad stride or alignment */
  SLA_ERR_UNSUPPORTED = 2,   /* d, block size or precision this build does not implement */
  SLA_ERR_WORKSPACE = 3,     /* workspace NULL, too small or misaligned */
  SLA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (launch, encode) */
  SLA_ERR_DEVICE_TIMEOUT = 5,/* a kernel gave up waiting (device error word) */
  SLA_ERR_DEVICE_BAD_INDEX = 6 /* a kernel met a LUT index out of range */
} sla_status_t;

typedef enum {
  SLA_COMBINE_PROJ = 0,  /* [SLA] Eq. 6:  O = O^s + Proj(O^l), Proj(x) = x W^T + b */
  SLA_COMBINE_ALPHA = 1  /* [SLA2] §3:    O = alpha_h O^s + (1 - alpha_h) O^l       */
} sla_combine_t;

typedef enum {
  SLA_QK_BF16 = 0,      /* Q K^T of critical blocks in bf16, fp32 accumulate */
  SLA_QK_FP8_E4M3 = 1,  /* [SLA2] §5: Q, K quantised to E4M3 with one scale per
                           64-row block (max|x|/448) before Q K^T */
  SLA_QK_INT8 = 2       /* [SLA2] §5 (low-bit tensors "such as INT8 or FP8"): Q, K
                           quantised to symmetric INT8 codes in [-127, 127] with one
                           scale per 64-row block (max|x|/127), integer Q K^T with
                           int32 accumulation, rescaled by the two block scales */
} sla_qk_prec_t;

typedef enum {
  SLA_PV_BF16 = 0,      /* P V of critical blocks in bf16, fp32 accumulate */
  SLA_PV_FP8_E4M3 = 1   /* [SLA2] §5: P and V quantised to E4M3, product dequantised:
                           P = 2^(s log2 e - M) with M the row maximum rounded up to
                           whole log2 units, stored as E4M3(448 P); V with one scale
                           per (head, channel) max|V[:, c]| / 448 */
} sla_pv_prec_t;

typedef enum {
  SLA_PHI_SOFTMAX = 0,  /* phi(x) = softmax of x over the head dimension ([SLA] Fig. 4) */
  SLA_PHI_ELU1 = 1      /* phi(x) = elu(x) + 1, the ablation of [SLA] Table 2 */
} sla_phi_t;

typedef struct {
  int B, H, N, d;      /* batch, heads, tokens, head dimension */
  int b_q, b_kv;       /* query / key-value block sizes ([SLA] §4 notation: 64) */
  float k_h;           /* critical fraction per row (top k_h%, [SLA] §2 Q2 step 2) */
  float k_l;           /* negligible fraction per row (bottom k_l%) */
  int combine;         /* sla_combine_t */
  int qk_prec;         /* sla_qk_prec_t */
  int smooth_k;        /* 1: subtract the token mean of K before mask prediction
                          ([SLA] §7 item 3); it cannot change a row-wise ranking */
  float eps;           /* added to the linear-branch denominator ([SLA] §4 check 5) */
  int64_t stride_q[3]; /* element strides of Q for the B, H, N dimensions */
  int64_t stride_k[3];
  int64_t stride_v[3];
  int64_t stride_o[3];
  int phi;             /* sla_phi_t: the linear branch's feature map, for K and Q */
  int linear_over_all; /* 1: H_i, Z_i sum h_j, z_j over every key block instead of the
                          marginal ones (the released code's variant, [SLA] §7 item 2) */
  int pv_prec;         /* sla_pv_prec_t (FP8: d = 128 only) */
} sla_params_t;

/* Fills a params struct for contiguous [B,H,N,d] tensors, b = 64, eps = 1e-5,
 * bf16 Q K^T and P V, softmax feature map, linear branch over the marginal blocks. */
void sla_params_default(sla_params_t* p, int B, int H, int N, int d, float k_h, float k_l,
                        int combine);

/* Block counts per row: n_h = max(1, floor(k_h*T_kv + 1e-9)),
 * n_l = min(floor(k_l*T_kv + 1e-9), T_kv - n_h).  The pages give "top k_h%"
 * and "bottom k_l%" per row without a rounding rule; flooring keeps at least
 * the stated sparsity and one critical block keeps the sparse softmax defined.
 * Any output pointer may be NULL. */
sla_status_t sla_block_counts(const sla_params_t* p, int* T_q, int* T_kv, int* n_h, int* n_l);

/* Bytes of device workspace the calls below need (the same size serves all
 * of them, including sla_attention). */
sla_status_t sla_workspace_size(const sla_params_t* p, size_t* bytes);

/* Bytes of the caller-owned linear statistics buffer `hz`:
 * bf16 [B*H][T_kv][d*d + d]. */
sla_status_t sla_hz_size(const sla_params_t* p, size_t* bytes);

/*
 * Compressed mask prediction ([SLA] §2 Q2 steps 1-2, Fig. 4 left; [SLA2] §4).
 *   Q_c = mean_pool(Q), K_c = mean_pool(K) over blocks of b_q / b_kv tokens;
 *   SLA2 router: Q_c <- Q_c Wq^T, K_c <- K_c Wk^T (Wq, Wk fp32 [d][d],
 *   shared by all heads, no bias; NULL = identity, which is SLA);
 *   logits = Q_c K_c^T / sqrt(d); P_c = row softmax (monotone, so the
 *   selection ranks logits directly).  Per row: the n_h highest blocks are
 *   critical (1), the n_l lowest negligible (-1), the rest marginal (0); ties
 *   rank the lower block index first.
 * Outputs (device, caller-allocated):
 *   mc  int8  [B*H][T_q][T_kv]   values in {1, 0, -1}
 *   lut int32 [B*H][T_q][n_h]    critical block indices in ascending order
 */
sla_status_t sla_predict_mask(const sla_params_t* p, const void* Q, const void* K,
                              const float* Wq, const float* Wk, int8_t* mc, int32_t* lut,
                              void* workspace, size_t workspace_bytes, sla_stream_t stream);

/*
 * The router's compressed attention ([SLA2] §4 Learnable Router; [SLA] Fig. 4):
 * P_c = row softmax of the logits that sla_predict_mask ranks (the same pooling,
 * smooth-K and Wq / Wk projections, the same fp32 logits).
 * Output (device, caller-allocated, 16-byte aligned):
 *   Pc  fp32 [B*H][T_q][T_kv]
 * Uses the workspace of sla_workspace_size.  Errors: SLA_ERR_INVALID_ARG for
 * NULL or misaligned pointers, SLA_ERR_WORKSPACE, SLA_ERR_CUDA.
 */
sla_status_t sla_router_probs(const sla_params_t* p, const void* Q, const void* K,
                              const float* Wq, const float* Wk, float* Pc, void* workspace,
                              size_t workspace_bytes, sla_stream_t stream);

/*
 * SoftTop-k, the training-time replacement of the router's hard row-wise Top-k
 * ([SLA2] §4 Learnable Router, §6 Training with SLA2):
 *   M[i][j] = sigmoid((Pc[i][j] - lambda_i) / tau),
 * lambda_i chosen per row by bisection so that sum_j M[i][j] = n_h (the hard
 * Top-k's count, sla_block_counts), 40 halvings of [min Pc - 50 tau,
 * max Pc + 50 tau] in fp32.  As tau -> 0, M becomes the hard mask's critical
 * set.  The pages fix the sigmoid, tau, the binary search and the row sum;
 * the target n_h and the input P_c are this library's readings.
 * Inputs (device): Pc fp32 [B*H][T_q][T_kv] (e.g. from sla_router_probs), tau > 0.
 * Outputs (device, caller-allocated): M fp32 [B*H][T_q][T_kv], lambda fp32
 * [B*H][T_q].  Pc and M 16-byte aligned.  No workspace.
 * Errors: SLA_ERR_INVALID_ARG (NULL or misaligned pointers, tau not a finite
 * number >= FLT_MIN, the smallest normal fp32 value), SLA_ERR_CUDA.
 */
sla_status_t sla_soft_topk(const sla_params_t* p, const float* Pc, float tau, float* M,
                           float* lambda, sla_stream_t stream);

/*
 * Per-key-block linear-attention statistics ([SLA] §2 Q2 step 3, Fig. 4
 * "Linear Attention Precomputation"):
 *   h_j = phi(K_j)^T V_j  (d x d),   z_j = rowsum(phi(K_j)^T)  (d),
 * phi = softmax over the head dimension (elu + 1 with phi = SLA_PHI_ELU1),
 * only real tokens of a partial block.
 * For the SLA combine, Proj's weight (fp32 [d][d], nn.Linear convention) is
 * folded in: h_j W^T is stored, which is exact by linearity because
 * Proj(O^l) = (phi(Q) H / den) W^T + b = phi(Q) (H W^T) / den + b.  Pass
 * proj_w = NULL for SLA2 (or Proj = identity).
 * Output hz (device, caller-allocated, sla_hz_size bytes): bf16
 *   [B*H][T_kv][d*d + d]: element (b*d + a) holds (h_j W^T)[a][b] (the
 *   transpose, row b contiguous in a), element d*d + a holds z_j[a].
 */
sla_status_t sla_precompute_linear(const sla_params_t* p, const void* K, const void* V,
                                   const float* proj_w, void* hz, void* workspace,
                                   size_t workspace_bytes, sla_stream_t stream);

/*
 * The fused forward given a mask ([SLA] §2 Q2 steps 3-4, Fig. 4 right):
 * for every query block i
 *   O^s_i = softmax attention over the tokens of its critical blocks (lut),
 *           computed block by block with an online softmax;
 *   H_i = sum of h_j, Z_i = sum of z_j over its marginal blocks (mc == 0;
 *         every block with linear_over_all);
 *   O^l_i = phi(Q_i) H_i / (phi(Q_i) Z_i + eps)        ([SLA] Eq. 3-4);
 *   negligible blocks (mc == -1) are never read;
 *   SLA:  O = O^s + O^l W^T + proj_b  (W folded into hz; proj_b fp32 [d] or NULL)
 *   SLA2: O = alpha[b*H+h] O^s + (1 - alpha[b*H+h]) O^l  (alpha fp32 [B*H])
 * mc and lut must come from sla_predict_mask with the same params (or obey
 * its contract: n_h ascending in-range indices per row, consistent with mc).
 * O is bf16 [B,H,N,d] (strides from params).
 */
sla_status_t sla_forward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                         const int8_t* mc, const int32_t* lut, const void* hz,
                         const float* proj_b, const float* alpha, void* O, void* workspace,
                         size_t workspace_bytes, sla_stream_t stream);

/*
 * sla_forward that also keeps what sla_backward needs (device, caller-allocated):
 *   lse       fp32 [B*H][N]: per query row, log(sum over its critical tokens t of
 *             exp(q_n . k_t / sqrt(d))) (natural log);
 *   o_sparse  fp32 [B*H][N][d]: the sparse branch's output o^s of every row (the
 *             backward needs it apart from the combined O, in full precision).
 */
sla_status_t sla_forward_train(const sla_params_t* p, const void* Q, const void* K,
                               const void* V, const int8_t* mc, const int32_t* lut,
                               const void* hz, const float* proj_b, const float* alpha, void* O,
                               float* lse, float* o_sparse, void* workspace,
                               size_t workspace_bytes, sla_stream_t stream);

/*
 * The two halves of sla_forward, for callers that schedule or time them
 * separately (sla_forward is exactly sla_aggregate_marginal followed by
 * sla_fused_forward on the same stream and workspace).
 *
 * sla_aggregate_marginal: for every query block i, [H_i^T | Z_i] = sum over
 * its marginal blocks (mc == 0; every block with linear_over_all) of
 * [h_j^T | z_j] ([SLA] §2 Q2 step 3,
 * marginal blocks accumulate h_j and z_j), computed as one 0/1-matrix product per head on
 * the tensor cores; the result stays in the workspace.
 *
 * sla_fused_forward: the per-query-block kernel (sparse branch over the
 * critical blocks of lut, linear branch from the workspace's [H_i^T | Z_i],
 * combine), writing O.  Requires a preceding sla_aggregate_marginal on the
 * same workspace.
 */
sla_status_t sla_aggregate_marginal(const sla_params_t* p, const int8_t* mc, const void* hz,
                                    void* workspace, size_t workspace_bytes, sla_stream_t stream);
sla_status_t sla_fused_forward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                               const int32_t* lut, const float* proj_b, const float* alpha,
                               void* O, void* workspace, size_t workspace_bytes,
                               sla_stream_t stream);

/*
 * The two steps of sla_fused_forward, for callers that time or schedule them
 * apart (sla_fused_forward is exactly sla_pair_query_blocks followed by
 * sla_fused_forward_paired on the same stream and workspace).
 *
 * sla_pair_query_blocks: chooses which two query blocks of a head share one
 * 128-row tile of the fused kernel, from lut (blocks whose critical lists
 * overlap most are paired, so the union of the two lists is small).  A pure
 * scheduling choice: any pairing gives the same output.  The pairs stay in the
 * workspace, int2 [B*H][ceil(T_q / 2)] (second block -1: a tile with one
 * block) at the offset sla_workspace_pairs returns.
 *
 * sla_fused_forward_paired: the fused kernel on the pairs already in the
 * workspace (requires sla_aggregate_marginal and sla_pair_query_blocks, in
 * either order, on the same workspace and lut).
 *
 * sla_workspace_pairs: byte offset of the pairs in the workspace and their
 * number (B*H*ceil(T_q / 2)), for callers that read them back.
 * Errors: SLA_ERR_INVALID_ARG (NULL pointers), SLA_ERR_WORKSPACE, SLA_ERR_CUDA.
 */
sla_status_t sla_pair_query_blocks(const sla_params_t* p, const int32_t* lut, void* workspace,
                                   size_t workspace_bytes, sla_stream_t stream);
sla_status_t sla_fused_forward_paired(const sla_params_t* p, const void* Q, const void* K, const void* V,
                                      const int32_t* lut, const float* proj_b, const float* alpha,
                                      void* O, void* workspace, size_t workspace_bytes,
                                      sla_stream_t stream);
sla_status_t sla_workspace_pairs(const sla_params_t* p, size_t* offset, size_t* count);

/*
 * The whole forward in one call: sla_predict_mask, sla_precompute_linear and
 * sla_forward, with mc, lut and hz kept in the workspace
 * (sla_attention_workspace_size bytes).  proj_w / proj_b are used by the SLA
 * combine, Wq / Wk / alpha by SLA2 (Wq, Wk may be NULL).  The linear
 * statistics (sla_precompute_linear) run on a second stream that the library
 * creates once per device (with two events; no device memory), beside mask
 * prediction and the pairing of query blocks on `stream`; everything is
 * ordered after the work already on `stream`, and `stream` waits for the
 * second stream before the aggregation, so the call behaves as if all of it
 * ran on `stream`.  Calls from several host threads serialise their enqueueing
 * on that stream.  Under stream capture everything runs on `stream` in order.
 */
sla_status_t sla_attention_workspace_size(const sla_params_t* p, size_t* bytes);
sla_status_t sla_attention(const sla_params_t* p, const void* Q, const void* K, const void* V,
                           const float* proj_w, const float* proj_b, const float* alpha,
                           const float* Wq, const float* Wk, void* O, void* workspace,
                           size_t workspace_bytes, sla_stream_t stream);

/*
 * sla_attention with the activations in host memory: copies Q, K, V (host,
 * contiguous [B,H,N,d] bf16; page-locked memory makes the copies
 * asynchronous) into device staging buffers inside the workspace, runs the
 * forward and copies O back to O_host.  The (batch, head) problems are split
 * into up to 6 chunks that are pipelined: chunk c + 1 is copied in while chunk
 * c is computed on `stream` and chunk c - 1 is copied out, on two copy streams
 * the library creates once per device (with their events; no device memory).
 * Everything is ordered after the work already enqueued on `stream`, and
 * `stream` waits for the last copy, so O_host is valid once `stream` has been
 * synchronised.  The parameters proj_w, proj_b, alpha, Wq, Wk stay device
 * pointers.  The params' strides must describe contiguous tensors.  Calls that
 * overlap on one device must use different workspaces and may not run
 * concurrently (the copy streams are shared).
 */
sla_status_t sla_attention_host_workspace_size(const sla_params_t* p, size_t* bytes);
sla_status_t sla_attention_host(const sla_params_t* p, const void* Q_host, const void* K_host,
                                const void* V_host, const float* proj_w, const float* proj_b,
                                const float* alpha, const float* Wq, const float* Wk,
                                void* O_host, void* workspace, size_t workspace_bytes,
                                sla_stream_t stream);

/*
 * sla_predict_mask without a workspace argument.  The pages describe no such
 * call: it exists for callers that cannot allocate device memory when they
 * predict the mask (allocation-free hot loops, host callbacks, memory planned
 * up front by an arena the caller does not own).  Its scratch (error word,
 * pooled / routed Q and K blocks, logit keys) lives in one static device array of
 * SLA_NOALLOC_SCRATCH_BYTES that every GPU using the library holds until the
 * process exits.  Inputs, outputs and results are those of sla_predict_mask.
 *   - Problems whose scratch exceeds the array (B*H*T_q*T_kv*4 bytes of
 *     logit keys plus B*H*(T_q + T_kv)*d*4, twice the latter plus B*H*d*4
 *     with a router or smooth-K, plus 256) return SLA_ERR_WORKSPACE before
 *     any launch.
 *   - The first call on a device looks up the array's address on that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     race and must be serialised by the caller.
 *   - Nothing is allocated; the error word is cleared with cudaMemsetAsync.
 */
#define SLA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
sla_status_t sla_predict_mask_noalloc(const sla_params_t* p, const void* Q, const void* K,
                                      const float* Wq, const float* Wk, int8_t* mc,
                                      int32_t* lut, sla_stream_t stream);

/*
 * Backward of sla_forward_train ([SLA2] App. A; [SLA] §4 check 6): the
 * gradients of L = sum(O * dO) for fixed mc (hard Top-k has no gradient).
 * SLA2's router is trained through SoftTop-k; its forward is sla_soft_topk,
 * but its gradient is not built, so Wq / Wk get no gradient here.
 *   sparse branch  the FlashAttention backward over the critical blocks only:
 *                  P = exp(q.k / sqrt(d) - lse), dS = P (dP - D) with
 *                  D_r = dO^s_r . o^s_r; one kernel for dQ (per query-block
 *                  pair, over its critical lists) and one for dK, dV (per
 *                  key-block pair, over the query blocks that have it critical);
 *   linear branch  per query block dH_i, dZ_i, summed into every marginal key
 *                  block's dh_j, dz_j (the forward's 0/1 product, transposed),
 *                  then back through h_j = phi(K_j)^T V_j, z_j and phi;
 *   combine        SLA: dO^s = dO, the linear branch sees dO W;
 *                  dproj_w = dO^T o_l, dproj_b = sum dO.
 *                  SLA2: dO^s = alpha dO, dO^l = (1 - alpha) dO,
 *                  dalpha = sum (o^s - o^l) . dO per head.
 * Inputs (device): Q, K, V and params as given to the forward; mc, lut from
 *   sla_predict_mask; hz from sla_precompute_linear (Proj's W folded in for
 *   SLA); proj_w fp32 [d][d] (SLA), proj_b fp32 [d] or NULL (SLA), alpha fp32
 *   [B*H] (SLA2); o_sparse and lse from sla_forward_train; dO bf16 [B,H,N,d]
 *   with the strides of O (stride_o).
 * Outputs (device, caller-allocated, overwritten): dQ, dK, dV bf16 with the
 *   strides of Q, K, V; dproj_w fp32 [d][d] and dproj_b fp32 [d] (SLA; either
 *   may be NULL); dalpha fp32 [B*H] (SLA2; may be NULL).
 * Workspace: sla_backward_workspace_size bytes, 256-byte aligned; its first
 *   word is the device error word (zero it once; sla_get_device_status reads
 *   and clears it).  Q K^T is recomputed in bf16 also when the forward ran
 *   it on 8-bit codes ([SLA2] §5 keeps the backward in full precision).
 */
sla_status_t sla_backward_workspace_size(const sla_params_t* p, size_t* bytes);
sla_status_t sla_backward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                          const int8_t* mc, const int32_t* lut, const void* hz,
                          const float* proj_w, const float* proj_b, const float* alpha,
                          const float* o_sparse, const float* lse, const void* dO, void* dQ,
                          void* dK, void* dV, float* dproj_w, float* dproj_b, float* dalpha,
                          void* workspace, size_t workspace_bytes, sla_stream_t stream);

/*
 * Diagnostic (no counterpart on the pages): launches one thread that waits on a
 * barrier nothing completes.  The wait gives up after one second, records a
 * timeout in the error word of `workspace` (any workspace of this library, or
 * 256 zeroed bytes) and the kernel returns; sla_get_device_status then reports
 * SLA_ERR_DEVICE_TIMEOUT.  It exercises the failure path that every wait of
 * every kernel takes, without faulting the GPU.
 */
sla_status_t sla_selftest_wait_timeout(void* workspace, sla_stream_t stream);

/* Reads the device error word of `workspace` (synchronises `stream`) and
 * clears it.  Returns SLA_OK, SLA_ERR_DEVICE_TIMEOUT or
 * SLA_ERR_DEVICE_BAD_INDEX; *detail (may be NULL) receives the raw code. */
sla_status_t sla_get_device_status(void* workspace, sla_stream_t stream, int* detail);

/* Human-readable name of a status code (static storage). */
const char* sla_status_string(sla_status_t s);

/* Version of this ABI (major * 100 + minor). */
int sla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
