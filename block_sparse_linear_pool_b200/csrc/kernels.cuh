// Kernel argument blocks and host launchers of the SLA forward path.
#pragma once
#include "sm100.cuh"

namespace sla {

struct PoolArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  int64_t sq[3];  // element strides of Q for B, H, N
  int64_t sk[3];
  float* Qc;
  float* Kc;
  int H, N, T, bs;
};

struct SelectArgs {
  const float* Qc;  // [BH][Tq][d] pooled (and routed) queries
  const float* Kc;  // [BH][Tkv][d]
  uint32_t* keys;   // [BH][Tq][Tkv] scratch: order-preserving logit keys
  int8_t* mc;       // [BH][Tq][Tkv]
  int32_t* lut;     // [BH][Tq][nh]
  int d, Tq, Tkv, nh, nl, BH;
};

struct LogitArgs {
  const float* Qc;
  const float* Kc;
  uint32_t* keys;
  int d, Tq, Tkv;
};

struct KvPrepArgs {
  const float* proj_w;   // [d][d] fp32 or nullptr (identity)
  __nv_bfloat16* hz;     // [BH][Tkv][d*d + d]
  int* err;
  int H, N, Tkv, nitems;
  int phi;               // 0 softmax over d, 1 elu + 1
};

struct MargArgs {
  __nv_bfloat16* Hout;   // [BH][Tq][NN]
  int* err;
  int Tq, Tkv, NN, ktiles, BH;
  const int8_t* mc;      // [BH][Tq][Tkv] M_c (the TMEM-operand kernel builds its 0/1 rows from it)
  int all;               // every block counts (linear branch over all blocks)
};

struct QuantArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  int64_t sq[3];       // element strides of Q for B, H, N
  int64_t sk[3];
  uint8_t* Q8;         // [BH][T_q*64][d] e4m3
  uint8_t* K8;         // [BH][T_kv*64][d] e4m3
  float* scale_q;      // [BH][T_q]
  float* scale_k;      // [BH][T_kv]
  int H, N, Tq, Tkv;
  int int8;            // 1: symmetric INT8 codes (scale max/127), 0: E4M3 (scale max/448)
};

struct FusedArgs {
  const int32_t* lut;     // [BH][Tq][nh]
  const __nv_bfloat16* Hz;  // [BH][Tq][NN] aggregated H_i^T and Z_i
  const float* proj_b;    // [d] or nullptr
  const float* alpha;     // [BH] or nullptr
  __nv_bfloat16* O;
  int* err;
  int64_t so0, so1, so2;  // O strides (elements) for B, H, N
  int H, N, Tq, Tkv, nh, NN;
  int combine;            // 0 proj, 1 alpha
  float scale_log2;       // log2(e) / sqrt(d)
  float eps;
  const float* scale_q;   // 8-bit Q K^T: per (head, query block) scale of Q, else nullptr
  const float* scale_k;   // 8-bit Q K^T: per (head, key block) scale of K, else nullptr
  int phi;                // 0 softmax over d, 1 elu + 1
  float* lse;             // [BH][N] natural-log sum of exp of the scaled critical scores, or nullptr
  float* os;              // [BH][N][d] the sparse branch's output o^s (fp32), or nullptr
  const unsigned int* vmax;  // FP8 P V: per (head, channel) max |V| (float bits), else nullptr
  const int2* pairs;      // [BH][ceil(Tq / 2)] the two query blocks of each CTA (b = -1: none)
  const uint16_t* ulist;  // persistent kernel: per tile the union record (tile_union_kernel)
  int urec;               // uint16 per union record
  int BH;
};

// ---- backward
struct BwdRowsArgs {
  const __nv_bfloat16* Q;
  int64_t sq[3];
  const float* os;          // [BH][N][d] the forward's sparse-branch output (fp32)
  const __nv_bfloat16* dO;
  int64_t so[3];            // strides of dO
  const __nv_bfloat16* hagg;  // [BH][Tq][NN] forward's [H'_i^T | Z_i]
  const float* alpha;       // [BH] (SLA2) or nullptr
  const float* lse;         // [BH][N] from the forward
  float2* ld2;              // [BH][T_q * 64] out: (-lse * log2 e, -D), D = dO^s . o^s; (-inf, 0) past N
  float* dq_lin;            // [BH][N][d] out
  __nv_bfloat16* dhz;       // [BH][Tq][NN] out: [dH'_i^T | dZ_i]
  float* dalpha;            // [BH] accumulated (SLA2) or nullptr
  float* dproj_b;           // [d] accumulated (SLA) or nullptr
  int H, N, Tq, NN, combine, phi;
  float eps;
};

struct BwdKeysArgs {
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t sk[3], sv[3];
  const float* proj_w;      // [d][d] (SLA) or nullptr (identity)
  const __nv_bfloat16* dhz; // [BH][Tkv][NN] [dh'_j^T | dz_j]
  float* dk_lin;            // [BH][N][d] out
  float* dv_lin;            // [BH][N][d] out
  float* dproj_w;           // [d][d] accumulated (SLA) or nullptr
  int BH, H, N, Tkv, NN, phi;
};

struct BwdSparseArgs {
  const int32_t* lut;       // [BH][Tq][nh]
  const int32_t* rptr;      // [BH][Tkv + 1] reverse lists: query blocks with j critical
  const int32_t* rows;      // [BH][Tq * nh]
  const float2* ld2;        // [BH][T_q * 64] (-lse * log2 e, -D) per query row, padded rows (-inf, 0)
  const float* alpha;       // [BH] (SLA2) or nullptr
  const float* q_lin;       // [BH][N][d] dq (linear part), or dk (linear) for the key kernel
  const float* v_lin;       // [BH][N][d] dv (linear part) for the key kernel
  const int2* pairs;        // [BH][ceil(T / 2)] block pairs: query blocks (dQ) or key blocks (dK / dV)
  __nv_bfloat16* out0;      // dQ, or dK for the key kernel
  __nv_bfloat16* out1;      // dV for the key kernel
  int64_t s0[3], s1[3];     // strides of out0, out1
  int* err;
  int H, N, Tq, Tkv, nh, combine;
  float scale_log2;         // log2(e) / sqrt(d)
  float scale;              // 1 / sqrt(d)
};

cudaError_t launch_bwd_rows(const BwdRowsArgs& a, int D, int BH, cudaStream_t s);
cudaError_t launch_bwd_keys(const BwdKeysArgs& a, int D, cudaStream_t s);
cudaError_t launch_bwd_rows_tc(const CUtensorMap& mapH, const CUtensorMap& mapZ, const BwdRowsArgs& a,
                               int* err, int BH, cudaStream_t s);
cudaError_t launch_bwd_keys_tc(const CUtensorMap& mapG, const CUtensorMap& mapZ, const CUtensorMap& mapK2,
                               const CUtensorMap& mapV2, const BwdKeysArgs& a, __nv_bfloat16* ubuf, int* err,
                               cudaStream_t s);
cudaError_t launch_dw(const CUtensorMap& mapU, const CUtensorMap& mapV2, int H, int BH, int Tkv, float* dW,
                      int* err, cudaStream_t s);
cudaError_t launch_colsum(const __nv_bfloat16* dO, const int64_t* so, int H, int N, int BH, int D,
                          float* out, cudaStream_t s);
cudaError_t launch_rlut(const int8_t* mc, int32_t* rcnt, int32_t* rptr, int32_t* rows, int BH,
                        int Tq, int Tkv, int nh, cudaStream_t s);
cudaError_t launch_bwd_dq(const CUtensorMap& mapQ, const CUtensorMap& mapdO, const CUtensorMap& mapK,
                          const CUtensorMap& mapV, const BwdSparseArgs& a, int D, int BH,
                          cudaStream_t s);
cudaError_t launch_bwd_dkdv(const CUtensorMap& mapK2, const CUtensorMap& mapV2,
                            const CUtensorMap& mapQ1, const CUtensorMap& mapdO1,
                            const BwdSparseArgs& a, int D, int BH, cudaStream_t s);

cudaError_t launch_pool(const PoolArgs& a, int D, int BH, cudaStream_t s);
cudaError_t launch_logits(const LogitArgs& a, int BH, cudaStream_t s);
cudaError_t launch_router_probs(const uint32_t* keys, float* Pc, int Tkv, int64_t rows, cudaStream_t s);
cudaError_t launch_soft_topk(const float* Pc, float* M, float* lam, int Tkv, int64_t rows, int nh, float tau,
                             cudaStream_t s);
// ov: scratch of pairing_overlap_bytes(BH, T); ncol: the range of the list entries
size_t pairing_overlap_bytes(int BH, int T);
cudaError_t launch_pairing(const int32_t* lut, int BH, int Tq, int nh, int ncol, uint16_t* ov, int2* pairs,
                           cudaStream_t s);
cudaError_t launch_pairing_csr(const int32_t* rows, const int32_t* ptr, int64_t stride, int BH, int T,
                               int ncol, uint16_t* ov, int2* pairs, cudaStream_t s);
cudaError_t launch_router(const float* Qc, const float* Kc, float* Qr, float* Kr, float* kmean,
                          const float* Wq, const float* Wk, bool smooth, int BH, int Tq, int Tk,
                          int N, int bs, int D, cudaStream_t s);
size_t select_smem_bytes(int Tk);
cudaError_t launch_select(const SelectArgs& a, int BH, cudaStream_t s);

// mapO: hz viewed as (a: d, b: d, j: T_kv, bh) tiles of 64 x d for TMA stores.
cudaError_t launch_kv_prep(const CUtensorMap& mapK, const CUtensorMap& mapV, const CUtensorMap& mapO,
                           const KvPrepArgs& a, int D, cudaStream_t s, int ctas_per_sm = 2);

cudaError_t launch_marg_matrix(const int8_t* mc, __nv_bfloat16* mm, int BH, int Tq, int Tkv,
                               int Tkvp, bool all, cudaStream_t s);
cudaError_t launch_marg_matrix_t(const int8_t* mc, __nv_bfloat16* mt, int BH, int Tq, int Tkv,
                                 int Tqp, bool all, cudaStream_t s);
// mapO: the output rows [BH][M][NN] bf16, box 64 x 128, 128-byte swizzle (TMA stores)
// T_kv <= 512: the 0/1 operand lives in TMEM, built from M_c by the kernel itself.
constexpr int kMargTmemMaxTkv = 512;
cudaError_t launch_marg_gemm_tm(const CUtensorMap& mapB, const CUtensorMap& mapO, const MargArgs& a, int BH,
                                cudaStream_t s);
cudaError_t launch_marg_gemm(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapO,
                             const MargArgs& a,
                             int BH, cudaStream_t s);

cudaError_t launch_quant_fp8(const QuantArgs& a, int BH, cudaStream_t s);

// Per tile of the persistent fused kernel: the union of its two query blocks'
// critical lists (uint16 records of urec entries: count, then j | flag << 14 from 8).
cudaError_t launch_tile_union(const int32_t* lut, const int2* pairs, int BH, int Tq, int Tkv, int nh, int urec,
                              uint16_t* out, int* err, cudaStream_t s);
// The persistent fused kernel (bf16 Q K^T and P V, no training outputs); nsm = SM count.
cudaError_t launch_fused_pt(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                            const CUtensorMap& mapH, const CUtensorMap& mapZ, const FusedArgs& a, int D, int nsm,
                            cudaStream_t s);
size_t fused_pt_smem_bytes(int D, int urec);
// The split-union kernel: one tile per CTA, its steps alternating between two
// softmax warpgroups (bf16 Q K^T and P V); one CTA per SM.
cudaError_t launch_fused_sk(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                            const CUtensorMap& mapH, const FusedArgs& a, int D, int nsm, cudaStream_t s);
size_t fused_sk_smem_bytes(int D, int urec);
cudaError_t launch_vquant_fp8(const __nv_bfloat16* V, const int64_t* sv, int H, int N, int T, int BH, int D,
                              unsigned int* vmax, uint8_t* V8T, cudaStream_t s);

// qk8: 0 bf16 Q K^T, 1 E4M3, 2 INT8; mapQ8 / mapK8 are used only for qk8 != 0 (d = 128 only).
cudaError_t launch_fused(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                         const CUtensorMap& mapH, const CUtensorMap& mapZ, const CUtensorMap& mapQ8,
                         const CUtensorMap& mapK8, const FusedArgs& a, int D, int qk8, bool pv8, int BH,
                         cudaStream_t s);

}  // namespace sla
