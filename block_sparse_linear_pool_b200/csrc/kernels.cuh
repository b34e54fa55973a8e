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
  const float* scale_q;   // FP8 path: per (head, query block) scale of Q, else nullptr
  const float* scale_k;   // FP8 path: per (head, key block) scale of K, else nullptr
  int phi;                // 0 softmax over d, 1 elu + 1
};

cudaError_t launch_pool(const PoolArgs& a, int D, int BH, cudaStream_t s);
cudaError_t launch_router(const float* Qc, const float* Kc, float* Qr, float* Kr, float* kmean,
                          const float* Wq, const float* Wk, bool smooth, int BH, int Tq, int Tk,
                          int N, int bs, int D, cudaStream_t s);
size_t select_smem_bytes(int Tk);
cudaError_t launch_select(const SelectArgs& a, int BH, cudaStream_t s);

// mapO: hz viewed as (a: d, b: d, j: T_kv, bh) tiles of 64 x d for TMA stores.
cudaError_t launch_kv_prep(const CUtensorMap& mapK, const CUtensorMap& mapV, const CUtensorMap& mapO,
                           const KvPrepArgs& a, int D, cudaStream_t s);

cudaError_t launch_marg_matrix(const int8_t* mc, __nv_bfloat16* mm, int BH, int Tq, int Tkv,
                               int Tkvp, bool all, cudaStream_t s);
cudaError_t launch_marg_gemm(const CUtensorMap& mapA, const CUtensorMap& mapB, const MargArgs& a,
                             int BH, cudaStream_t s);

cudaError_t launch_quant_fp8(const QuantArgs& a, int BH, cudaStream_t s);

// mapQ8 / mapK8 are used only when fp8 is set (d = 128 only).
cudaError_t launch_fused(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                         const CUtensorMap& mapH, const CUtensorMap& mapZ, const CUtensorMap& mapQ8,
                         const CUtensorMap& mapK8, const FusedArgs& a, int D, bool fp8, int BH,
                         cudaStream_t s);

}  // namespace sla
