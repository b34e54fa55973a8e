// Host side of the C ABI declared in include/sla.h: argument validation,
// workspace layout, TMA descriptor encoding and kernel launches.  Nothing here
// allocates device memory or synchronises a stream (except
// sla_get_device_status).
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "sla.h"
#include "kernels.cuh"

using namespace sla;

namespace {

constexpr int kMaxN = 262144;
constexpr size_t kAlign = 256;

struct Plan {
  int B, H, N, d, BH, Tq, Tkv, nh, nl, NN, Tkvp;
  bool fp8;  // Q K^T on 8-bit codes (E4M3 or INT8) with per-block scales
  bool qk_int8;  // ... INT8 (else E4M3)
  bool pv8;  // P V on E4M3 (P on the fixed scale 448, V per (head, channel))
  int phi;   // sla_phi_t
  bool all;  // linear branch over every key block
};

inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// uint16 per tile-union record of the persistent fused kernel: count, 7 unused,
// then up to min(2 n_h, T_kv) entries, rounded up to 16 bytes
inline int union_record(const Plan& p) {
  const int cap = 2 * p.nh < p.Tkv ? 2 * p.nh : p.Tkv;
  return 8 + ((cap + 7) & ~7);
}

// The persistent fused kernel serves bf16 Q K^T and P V (the inference and the
// training forward) when two CTAs fit an SM (its shared memory holds the union
// records); the 8-bit paths and the rest use the per-tile kernel.
inline bool pt_eligible(const Plan& p) {
  return !p.fp8 && !p.pv8 && fused_pt_smem_bytes(p.d, union_record(p)) <= 113 * 1024;
}

// The split-union kernel (one tile per SM, two softmax warpgroups, a 6-stage
// ring) needs up to 227 KB of shared memory.
inline bool sk_eligible(const Plan& p) {
  return !p.fp8 && !p.pv8 && fused_sk_smem_bytes(p.d, union_record(p)) <= 227 * 1024;
}

// Which bf16 kernel schedule runs: the SLA_FUSED_SCHEDULE environment variable
// ("split" or "persistent") overrides the default (persistent), for comparisons.
// read at every call, so that a process can switch between the schedules
inline bool prefer_split() {
  const char* e = std::getenv("SLA_FUSED_SCHEDULE");
  return e && std::strcmp(e, "split") == 0;
}

// SLA_MARG_KERNEL=tmem selects, for T_kv <= 512, the aggregation GEMM whose
// 0/1 operand sits in TMEM; by default the one with both operands in shared
// memory runs (measured faster at the 1.3B shapes).
inline bool prefer_tmem_marg() {
  const char* e = std::getenv("SLA_MARG_KERNEL");
  return e && std::strcmp(e, "tmem") == 0;
}

struct Layout {
  size_t err, qc, kc, qr, kr, kmean, keys, mm, hagg;      // sla_workspace_size ...
  size_t q8, k8, scq, sck, v8t, vmax, pairs, pov, ulist, end;  // ... (+ 8-bit operands, tiles)
  size_t mc, lut, hz, end_attn;                           // + sla_attention extras
  size_t hq, hk, hv, ho, end_host;                        // + sla_attention_host staging
};

Layout layout_of(const Plan& p) {
  Layout L;
  size_t o = 0;
  L.err = o;   o = align_up(o + 256);
  L.qc = o;    o = align_up(o + (size_t)p.BH * p.Tq * p.d * 4);
  L.kc = o;    o = align_up(o + (size_t)p.BH * p.Tkv * p.d * 4);
  L.qr = o;    o = align_up(o + (size_t)p.BH * p.Tq * p.d * 4);
  L.kr = o;    o = align_up(o + (size_t)p.BH * p.Tkv * p.d * 4);
  L.kmean = o; o = align_up(o + (size_t)p.BH * p.d * 4);
  L.keys = o;  o = align_up(o + (size_t)p.BH * p.Tq * p.Tkv * 4);
  L.mm = o;    o = align_up(o + (size_t)p.BH * p.Tq * p.Tkvp * 2);
  L.hagg = o;  o = align_up(o + (size_t)p.BH * p.Tq * p.NN * 2);
  const size_t q8 = p.fp8 ? (size_t)p.BH * p.Tq * 64 * p.d : 0;
  const size_t k8 = p.fp8 ? (size_t)p.BH * p.Tkv * 64 * p.d : 0;
  L.q8 = o;    o = align_up(o + q8);
  L.k8 = o;    o = align_up(o + k8);
  L.scq = o;   o = align_up(o + (p.fp8 ? (size_t)p.BH * p.Tq * 4 : 0));
  L.sck = o;   o = align_up(o + (p.fp8 ? (size_t)p.BH * p.Tkv * 4 : 0));
  L.v8t = o;   o = align_up(o + (p.pv8 ? (size_t)p.BH * p.Tkv * p.d * 128 : 0));
  L.vmax = o;  o = align_up(o + (p.pv8 ? (size_t)p.BH * p.d * 4 : 0));
  L.pairs = o; o = align_up(o + (size_t)p.BH * ((p.Tq + 1) / 2) * 8);
  L.pov = o;   o = align_up(o + pairing_overlap_bytes(p.BH, p.Tq));
  L.ulist = o; o = align_up(o + (size_t)p.BH * ((p.Tq + 1) / 2) * union_record(p) * 2);
  L.end = o;
  L.mc = o;    o = align_up(o + (size_t)p.BH * p.Tq * p.Tkv);
  L.lut = o;   o = align_up(o + (size_t)p.BH * p.Tq * p.nh * 4);
  L.hz = o;    o = align_up(o + (size_t)p.BH * p.Tkv * p.NN * 2);
  L.end_attn = o;
  const size_t act = (size_t)p.BH * p.N * p.d * 2;
  L.hq = o;    o = align_up(o + act);
  L.hk = o;    o = align_up(o + act);
  L.hv = o;    o = align_up(o + act);
  L.ho = o;    o = align_up(o + act);
  L.end_host = o;
  return L;
}

void counts(int T, double kh, double kl, int* nh, int* nl) {
  int h = (int)std::floor(kh * T + 1e-9);
  if (h < 1) h = 1;
  if (h > T) h = T;
  int l = (int)std::floor(kl * T + 1e-9);
  if (l > T - h) l = T - h;
  if (l < 0) l = 0;
  *nh = h;
  *nl = l;
}

bool stride_ok(const int64_t* s, int d) {
  for (int i = 0; i < 3; ++i)
    if (s[i] <= 0 || (s[i] % 8) != 0) return false;
  return s[2] >= d;
}

sla_status_t make_plan(const sla_params_t* p, Plan* pl) {
  if (!p) return SLA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1) return SLA_ERR_INVALID_ARG;
  if (!(p->k_h >= 0.f && p->k_h <= 1.f && p->k_l >= 0.f && p->k_l <= 1.f)) return SLA_ERR_INVALID_ARG;
  if (!(p->eps >= 0.f) || !std::isfinite(p->eps)) return SLA_ERR_INVALID_ARG;
  if (p->combine != SLA_COMBINE_PROJ && p->combine != SLA_COMBINE_ALPHA) return SLA_ERR_INVALID_ARG;
  if (p->qk_prec != SLA_QK_BF16 && p->qk_prec != SLA_QK_FP8_E4M3 && p->qk_prec != SLA_QK_INT8)
    return SLA_ERR_INVALID_ARG;
  if (p->phi != SLA_PHI_SOFTMAX && p->phi != SLA_PHI_ELU1) return SLA_ERR_INVALID_ARG;
  if (p->linear_over_all != 0 && p->linear_over_all != 1) return SLA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if (p->qk_prec != SLA_QK_BF16 && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if (p->pv_prec != SLA_PV_BF16 && p->pv_prec != SLA_PV_FP8_E4M3) return SLA_ERR_INVALID_ARG;
  if (p->pv_prec == SLA_PV_FP8_E4M3 && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if (p->b_q != 64 || p->b_kv != 64) return SLA_ERR_UNSUPPORTED;
  if (p->N > kMaxN || (int64_t)p->B * p->H > 65535) return SLA_ERR_UNSUPPORTED;
  if (!stride_ok(p->stride_q, p->d) || !stride_ok(p->stride_k, p->d) ||
      !stride_ok(p->stride_v, p->d) || !stride_ok(p->stride_o, p->d))
    return SLA_ERR_INVALID_ARG;
  pl->B = p->B;
  pl->H = p->H;
  pl->N = p->N;
  pl->d = p->d;
  pl->BH = p->B * p->H;
  pl->Tq = (p->N + p->b_q - 1) / p->b_q;
  pl->Tkv = (p->N + p->b_kv - 1) / p->b_kv;
  counts(pl->Tkv, p->k_h, p->k_l, &pl->nh, &pl->nl);
  pl->NN = p->d * p->d + p->d;
  pl->Tkvp = (pl->Tkv + 7) & ~7;
  pl->fp8 = p->qk_prec != SLA_QK_BF16;
  pl->qk_int8 = p->qk_prec == SLA_QK_INT8;
  pl->pv8 = p->pv_prec == SLA_PV_FP8_E4M3;
  pl->phi = p->phi;
  pl->all = p->linear_over_all != 0;
  return SLA_OK;
}

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// rank-r tiled map (bf16 unless dt says otherwise), 128-byte swizzle (or none);
// dims/strides innermost first,
// strides in bytes for dims 1..r-1.
bool encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
            const uint64_t* strides, const uint32_t* box, bool swizzle = true,
            CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encoder();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  CUresult r = fn(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Q/K/V/O [B,H,N,d] with element strides s (B, H, N), box of `rows` tokens x 64 columns.
bool map_bhnd(CUtensorMap* m, const void* base, const Plan& p, const int64_t* s, int rows) {
  const uint64_t dims[4] = {(uint64_t)p.d, (uint64_t)p.N, (uint64_t)p.H, (uint64_t)p.B};
  const uint64_t strides[3] = {(uint64_t)s[2] * 2, (uint64_t)s[1] * 2, (uint64_t)s[0] * 2};
  const uint32_t box[4] = {64, (uint32_t)rows, 1, 1};
  return encode(m, base, 4, dims, strides, box);
}

sla_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA; }

#define SLA_TRY(x)                      \
  do {                                  \
    sla_status_t st_ = (x);             \
    if (st_ != SLA_OK) return st_;      \
  } while (0)

enum WsKind { WS_BASE, WS_ATTN, WS_HOST };

sla_status_t check_ws(const Plan& p, void* ws, size_t bytes, WsKind kind) {
  const Layout L = layout_of(p);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return SLA_ERR_WORKSPACE;
  const size_t need = kind == WS_BASE ? L.end : (kind == WS_ATTN ? L.end_attn : L.end_host);
  if (bytes < need) return SLA_ERR_WORKSPACE;
  return SLA_OK;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// a1 and the router part of a2: pooled (smoothed, projected) Q_c, K_c in the
// workspace; *qsrc, *ksrc point at the ones the logits use
sla_status_t router_inputs(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                           const float* Wq, const float* Wk, void* ws, cudaStream_t s,
                           const float** qsrc_out, const float** ksrc_out) {
  const Layout L = layout_of(pl);
  PoolArgs pa;
  pa.Q = static_cast<const __nv_bfloat16*>(Q);
  pa.K = static_cast<const __nv_bfloat16*>(K);
  for (int i = 0; i < 3; ++i) {
    pa.sq[i] = p->stride_q[i];
    pa.sk[i] = p->stride_k[i];
  }
  pa.Qc = at<float>(ws, L.qc);
  pa.Kc = at<float>(ws, L.kc);
  pa.H = pl.H;
  pa.N = pl.N;
  pa.T = pl.Tq;  // b_q == b_kv: T_q == T_kv
  pa.bs = 64;
  SLA_TRY(cuda_status(launch_pool(pa, pl.d, pl.BH, s)));
  const float* qsrc = pa.Qc;
  const float* ksrc = pa.Kc;
  if (Wq || Wk || p->smooth_k) {
    SLA_TRY(cuda_status(launch_router(pa.Qc, pa.Kc, at<float>(ws, L.qr), at<float>(ws, L.kr),
                                      at<float>(ws, L.kmean), Wq, Wk, p->smooth_k != 0, pl.BH,
                                      pl.Tq, pl.Tkv, pl.N, 64, pl.d, s)));
    qsrc = at<float>(ws, L.qr);
    ksrc = at<float>(ws, L.kr);
  }
  *qsrc_out = qsrc;
  *ksrc_out = ksrc;
  return SLA_OK;
}

sla_status_t predict_mask_impl(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                               const float* Wq, const float* Wk, int8_t* mc, int32_t* lut,
                               void* ws, cudaStream_t s) {
  const Layout L = layout_of(pl);
  const float *qsrc = nullptr, *ksrc = nullptr;
  SLA_TRY(router_inputs(pl, p, Q, K, Wq, Wk, ws, s, &qsrc, &ksrc));
  SelectArgs sa;
  sa.Qc = qsrc;
  sa.Kc = ksrc;
  sa.keys = at<uint32_t>(ws, L.keys);
  sa.mc = mc;
  sa.lut = lut;
  sa.d = pl.d;
  sa.Tq = pl.Tq;
  sa.Tkv = pl.Tkv;
  sa.nh = pl.nh;
  sa.nl = pl.nl;
  return cuda_status(launch_select(sa, pl.BH, s));
}

sla_status_t precompute_impl(const Plan& pl, const sla_params_t* p, const void* K, const void* V,
                             const float* proj_w, void* hz, void* ws, cudaStream_t s, int ctas_per_sm = 2) {
  CUtensorMap mk, mv, mo;
  if (!map_bhnd(&mk, K, pl, p->stride_k, 64) || !map_bhnd(&mv, V, pl, p->stride_v, 64))
    return SLA_ERR_CUDA;
  {
    const uint64_t dims[4] = {(uint64_t)pl.d, (uint64_t)pl.d, (uint64_t)pl.Tkv, (uint64_t)pl.BH};
    const uint64_t str[3] = {(uint64_t)pl.d * 2, (uint64_t)pl.NN * 2, (uint64_t)pl.Tkv * pl.NN * 2};
    const uint32_t box[4] = {64, (uint32_t)pl.d, 1, 1};
    if (!encode(&mo, hz, 4, dims, str, box)) return SLA_ERR_CUDA;
  }
  KvPrepArgs a;
  a.proj_w = (p->combine == SLA_COMBINE_PROJ) ? proj_w : nullptr;
  a.hz = static_cast<__nv_bfloat16*>(hz);
  a.err = at<int>(ws, layout_of(pl).err);
  a.H = pl.H;
  a.N = pl.N;
  a.Tkv = pl.Tkv;
  a.nitems = pl.BH * pl.Tkv;
  a.phi = pl.phi;
  return cuda_status(launch_kv_prep(mk, mv, mo, a, pl.d, s, ctas_per_sm));
}

// [BH][M][NN] bf16 rows as TMA store tiles of 64 columns x 128 rows (128-byte swizzle)
bool map_rows_out(CUtensorMap* m, void* base, int M, const Plan& pl) {
  const uint64_t dims[3] = {(uint64_t)pl.NN, (uint64_t)M, (uint64_t)pl.BH};
  const uint64_t str[2] = {(uint64_t)pl.NN * 2, (uint64_t)M * pl.NN * 2};
  const uint32_t box[3] = {64, 128, 1};
  return encode(m, base, 3, dims, str, box);
}

sla_status_t aggregate_impl(const Plan& pl, const int8_t* mc, const void* hz, void* ws,
                            cudaStream_t s) {
  const Layout L = layout_of(pl);
  if (pl.Tkv <= kMargTmemMaxTkv && prefer_tmem_marg()) {
    // the 0/1 rows are built from M_c inside the kernel, in TMEM
    CUtensorMap mb, mo;
    const uint64_t db[3] = {(uint64_t)pl.NN, (uint64_t)pl.Tkv, (uint64_t)pl.BH};
    const uint64_t sb[2] = {(uint64_t)pl.NN * 2, (uint64_t)pl.Tkv * pl.NN * 2};
    const uint32_t bb[3] = {64, 64, 1};
    if (!encode(&mb, hz, 3, db, sb, bb)) return SLA_ERR_CUDA;
    if (!map_rows_out(&mo, at<__nv_bfloat16>(ws, L.hagg), pl.Tq, pl)) return SLA_ERR_CUDA;
    MargArgs a;
    a.Hout = at<__nv_bfloat16>(ws, L.hagg);
    a.err = at<int>(ws, L.err);
    a.Tq = pl.Tq;
    a.Tkv = pl.Tkv;
    a.NN = pl.NN;
    a.ktiles = (pl.Tkv + 63) / 64;
    a.mc = mc;
    a.all = pl.all ? 1 : 0;
    return cuda_status(launch_marg_gemm_tm(mb, mo, a, pl.BH, s));
  }
  __nv_bfloat16* mm = at<__nv_bfloat16>(ws, L.mm);
  SLA_TRY(cuda_status(launch_marg_matrix(mc, mm, pl.BH, pl.Tq, pl.Tkv, pl.Tkvp, pl.all, s)));
  CUtensorMap ma, mb;
  const uint64_t da[3] = {(uint64_t)pl.Tkvp, (uint64_t)pl.Tq, (uint64_t)pl.BH};
  const uint64_t sa[2] = {(uint64_t)pl.Tkvp * 2, (uint64_t)pl.Tq * pl.Tkvp * 2};
  const uint32_t ba[3] = {64, 128, 1};
  const uint64_t db[3] = {(uint64_t)pl.NN, (uint64_t)pl.Tkv, (uint64_t)pl.BH};
  const uint64_t sb[2] = {(uint64_t)pl.NN * 2, (uint64_t)pl.Tkv * pl.NN * 2};
  const uint32_t bb[3] = {64, 64, 1};
  if (!encode(&ma, mm, 3, da, sa, ba) || !encode(&mb, hz, 3, db, sb, bb)) return SLA_ERR_CUDA;
  CUtensorMap mo;
  if (!map_rows_out(&mo, at<__nv_bfloat16>(ws, L.hagg), pl.Tq, pl)) return SLA_ERR_CUDA;
  MargArgs a;
  a.Hout = at<__nv_bfloat16>(ws, L.hagg);
  a.err = at<int>(ws, L.err);
  a.Tq = pl.Tq;
  a.Tkv = pl.Tkv;
  a.NN = pl.NN;
  a.ktiles = (pl.Tkv + 63) / 64;
  a.mc = nullptr;
  a.all = 0;
  return cuda_status(launch_marg_gemm(ma, mb, mo, a, pl.BH, s));
}

// out[bh][m][:] = sum_k A[bh][m][k] B[bh][k][:] for the 0/1 matrix A (bf16
// [BH][M][Kp], Kp = K rounded up to 8) and rows B (bf16 [BH][K][NN]).
sla_status_t zero_one_product(const Plan& pl, const __nv_bfloat16* A, int M, int Kdim, int Kp,
                              const void* B, __nv_bfloat16* out, int* err, cudaStream_t s) {
  CUtensorMap ma, mb;
  const uint64_t da[3] = {(uint64_t)Kp, (uint64_t)M, (uint64_t)pl.BH};
  const uint64_t sa[2] = {(uint64_t)Kp * 2, (uint64_t)M * Kp * 2};
  const uint32_t ba[3] = {64, 128, 1};
  const uint64_t db[3] = {(uint64_t)pl.NN, (uint64_t)Kdim, (uint64_t)pl.BH};
  const uint64_t sb[2] = {(uint64_t)pl.NN * 2, (uint64_t)Kdim * pl.NN * 2};
  const uint32_t bb[3] = {64, 64, 1};
  if (!encode(&ma, A, 3, da, sa, ba) || !encode(&mb, B, 3, db, sb, bb)) return SLA_ERR_CUDA;
  CUtensorMap mo;
  if (!map_rows_out(&mo, out, M, pl)) return SLA_ERR_CUDA;
  MargArgs a;
  a.Hout = out;
  a.err = err;
  a.Tq = M;
  a.Tkv = Kdim;
  a.NN = pl.NN;
  a.ktiles = (Kdim + 63) / 64;
  a.mc = nullptr;
  a.all = 0;
  return cuda_status(launch_marg_gemm(ma, mb, mo, a, pl.BH, s));
}

// which two query blocks share a tile; for the persistent kernel also each tile's union list
sla_status_t pairing_impl(const Plan& pl, const int32_t* lut, void* ws, cudaStream_t s) {
  const Layout L = layout_of(pl);
  int2* pairs = at<int2>(ws, L.pairs);
  SLA_TRY(cuda_status(launch_pairing(lut, pl.BH, pl.Tq, pl.nh, pl.Tkv, at<uint16_t>(ws, L.pov), pairs, s)));
  if (pt_eligible(pl) || sk_eligible(pl))
    SLA_TRY(cuda_status(launch_tile_union(lut, pairs, pl.BH, pl.Tq, pl.Tkv, pl.nh, union_record(pl),
                                          at<uint16_t>(ws, L.ulist), at<int>(ws, L.err), s)));
  return SLA_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

sla_status_t fused_impl(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                        const void* V, const int32_t* lut, const float* proj_b, const float* alpha,
                        void* O, void* ws, cudaStream_t s, float* lse = nullptr,
                        float* o_sparse = nullptr, bool pair = true) {
  const Layout L = layout_of(pl);
  __nv_bfloat16* hagg = at<__nv_bfloat16>(ws, L.hagg);
  CUtensorMap mq, mk, mv, mh, mz;
  if (!map_bhnd(&mq, Q, pl, p->stride_q, 64) || !map_bhnd(&mk, K, pl, p->stride_k, 64) ||
      !map_bhnd(&mv, V, pl, p->stride_v, 64))
    return SLA_ERR_CUDA;
  // which two query blocks share a CTA (similar critical lists: a smaller union)
  int2* pairs = at<int2>(ws, L.pairs);
  const bool pt = pt_eligible(pl);
  const bool sk = sk_eligible(pl) && (prefer_split() || !pt);
  if (pair) SLA_TRY(pairing_impl(pl, lut, ws, s));
  {
    // H_i^T as (a, b, i, bh) tiles of d x d; Z_i as one unswizzled row of d
    const uint64_t dh[4] = {(uint64_t)pl.d, (uint64_t)pl.d, (uint64_t)pl.Tq, (uint64_t)pl.BH};
    const uint64_t sh[3] = {(uint64_t)pl.d * 2, (uint64_t)pl.NN * 2,
                            (uint64_t)pl.Tq * pl.NN * 2};
    const uint32_t bxh[4] = {64, (uint32_t)pl.d, 1, 1};
    if (!encode(&mh, hagg, 4, dh, sh, bxh)) return SLA_ERR_CUDA;
    const uint64_t dz[3] = {(uint64_t)pl.NN, (uint64_t)pl.Tq, (uint64_t)pl.BH};
    const uint64_t sz[2] = {(uint64_t)pl.NN * 2, (uint64_t)pl.Tq * pl.NN * 2};
    const uint32_t bxz[3] = {64, 1, 1};
    if (!encode(&mz, hagg, 3, dz, sz, bxz, false)) return SLA_ERR_CUDA;
  }
  CUtensorMap mq8 = mq, mk8 = mk;  // placeholders unless the FP8 path runs
  const float* scq = nullptr;
  const float* sck = nullptr;
  if (pl.fp8) {
    QuantArgs qa;
    qa.Q = static_cast<const __nv_bfloat16*>(Q);
    qa.K = static_cast<const __nv_bfloat16*>(K);
    for (int i = 0; i < 3; ++i) {
      qa.sq[i] = p->stride_q[i];
      qa.sk[i] = p->stride_k[i];
    }
    qa.Q8 = at<uint8_t>(ws, L.q8);
    qa.K8 = at<uint8_t>(ws, L.k8);
    qa.scale_q = at<float>(ws, L.scq);
    qa.scale_k = at<float>(ws, L.sck);
    qa.H = pl.H;
    qa.N = pl.N;
    qa.Tq = pl.Tq;
    qa.Tkv = pl.Tkv;
    qa.int8 = pl.qk_int8 ? 1 : 0;
    SLA_TRY(cuda_status(launch_quant_fp8(qa, pl.BH, s)));
    const uint64_t dq[3] = {(uint64_t)pl.d, (uint64_t)pl.Tq * 64, (uint64_t)pl.BH};
    const uint64_t sq[2] = {(uint64_t)pl.d, (uint64_t)pl.Tq * 64 * pl.d};
    const uint32_t bq[3] = {(uint32_t)pl.d, 64, 1};
    const uint64_t dk[3] = {(uint64_t)pl.d, (uint64_t)pl.Tkv * 64, (uint64_t)pl.BH};
    const uint64_t sk[2] = {(uint64_t)pl.d, (uint64_t)pl.Tkv * 64 * pl.d};
    const uint32_t bk[3] = {(uint32_t)pl.d, 64, 1};
    if (!encode(&mq8, qa.Q8, 3, dq, sq, bq, true, CU_TENSOR_MAP_DATA_TYPE_UINT8) ||
        !encode(&mk8, qa.K8, 3, dk, sk, bk, true, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return SLA_ERR_CUDA;
    scq = qa.scale_q;
    sck = qa.scale_k;
  }
  const unsigned int* vmax = nullptr;
  if (pl.pv8) {
    // V^ [BH][T_kv][d rows][128 B] and the per-(head, channel) maxima
    uint8_t* v8t = at<uint8_t>(ws, L.v8t);
    unsigned int* vm = at<unsigned int>(ws, L.vmax);
    SLA_TRY(cuda_status(launch_vquant_fp8(static_cast<const __nv_bfloat16*>(V), p->stride_v, pl.H, pl.N,
                                          pl.Tkv, pl.BH, pl.d, vm, v8t, s)));
    const uint64_t dv[3] = {128, (uint64_t)pl.Tkv * pl.d, (uint64_t)pl.BH};
    const uint64_t sv[2] = {128, (uint64_t)pl.Tkv * pl.d * 128};
    const uint32_t bv[3] = {128, (uint32_t)pl.d, 1};
    if (!encode(&mv, v8t, 3, dv, sv, bv, true, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return SLA_ERR_CUDA;
    vmax = vm;
  }
  FusedArgs a;
  a.lut = lut;
  a.Hz = hagg;
  a.proj_b = (p->combine == SLA_COMBINE_PROJ) ? proj_b : nullptr;
  a.alpha = alpha;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.err = at<int>(ws, L.err);
  a.so0 = p->stride_o[0];
  a.so1 = p->stride_o[1];
  a.so2 = p->stride_o[2];
  a.H = pl.H;
  a.N = pl.N;
  a.Tq = pl.Tq;
  a.Tkv = pl.Tkv;
  a.nh = pl.nh;
  a.NN = pl.NN;
  a.combine = p->combine;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)pl.d));
  a.eps = p->eps;
  a.scale_q = scq;
  a.scale_k = sck;
  a.phi = pl.phi;
  a.lse = lse;
  a.os = o_sparse;
  a.vmax = vmax;
  a.pairs = pairs;
  a.ulist = at<uint16_t>(ws, L.ulist);
  a.urec = union_record(pl);
  a.BH = pl.BH;
  if (sk || pt) {
    const int nsm = sm_count();
    if (nsm <= 0) return SLA_ERR_CUDA;
    if (sk) return cuda_status(launch_fused_sk(mq, mk, mv, mh, a, pl.d, nsm, s));
    return cuda_status(launch_fused_pt(mq, mk, mv, mh, mz, a, pl.d, nsm, s));
  }
  const int qk8 = pl.fp8 ? (pl.qk_int8 ? 2 : 1) : 0;
  return cuda_status(launch_fused(mq, mk, mv, mh, mz, mq8, mk8, a, pl.d, qk8, pl.pv8, pl.BH, s));
}

sla_status_t forward_impl(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                          const void* V, const int8_t* mc, const int32_t* lut, const void* hz,
                          const float* proj_b, const float* alpha, void* O, void* ws,
                          cudaStream_t s, float* lse = nullptr, float* o_sparse = nullptr) {
  SLA_TRY(aggregate_impl(pl, mc, hz, ws, s));
  return fused_impl(pl, p, Q, K, V, lut, proj_b, alpha, O, ws, s, lse, o_sparse);
}

bool contiguous(const sla_params_t* p) {
  const int64_t s[3] = {(int64_t)p->H * p->N * p->d, (int64_t)p->N * p->d, (int64_t)p->d};
  for (int i = 0; i < 3; ++i)
    if (p->stride_q[i] != s[i] || p->stride_k[i] != s[i] || p->stride_v[i] != s[i] ||
        p->stride_o[i] != s[i])
      return false;
  return true;
}

// A second stream per device (no device memory), created once, for the part of
// the one-call forward that does not depend on the mask: the linear statistics
// (kv_prep) run beside mask prediction and the pairing of query blocks.
#ifndef SLA_OVERLAP_KV_CTAS_PER_SM
#define SLA_OVERLAP_KV_CTAS_PER_SM 1
#endif
struct SidePipe {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ok = false;
};
std::mutex& side_mutex() {
  static std::mutex m;
  return m;
}
// The caller holds side_mutex().
SidePipe* side_pipe() {
  static SidePipe pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SidePipe& sp = pipes[dev];
  if (!sp.ok) {
    if (cudaStreamCreateWithFlags(&sp.side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&sp.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&sp.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    sp.ok = true;
  }
  return &sp;
}

sla_status_t attention_impl(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                            const void* V, const float* proj_w, const float* proj_b,
                            const float* alpha, const float* Wq, const float* Wk, void* O,
                            void* ws, cudaStream_t s) {
  const Layout L = layout_of(pl);
  int8_t* mc = at<int8_t>(ws, L.mc);
  int32_t* lut = at<int32_t>(ws, L.lut);
  void* hz = at<void>(ws, L.hz);
  const bool alpha_mode = p->combine == SLA_COMBINE_ALPHA;
  const float* wq = alpha_mode ? Wq : nullptr;
  const float* wk = alpha_mode ? Wk : nullptr;
  const float* pw = alpha_mode ? nullptr : proj_w;
  // Under stream capture the side stream would join the caller's graph until
  // the capture ends: there everything runs in order on `s`.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return SLA_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) {
    SLA_TRY(predict_mask_impl(pl, p, Q, K, wq, wk, mc, lut, ws, s));
    SLA_TRY(precompute_impl(pl, p, K, V, pw, hz, ws, s));
    return forward_impl(pl, p, Q, K, V, mc, lut, hz, proj_b, alpha, O, ws, s);
  }
  sla_status_t st_kv = SLA_OK, st = SLA_OK;
  {
    std::lock_guard<std::mutex> lock(side_mutex());
    SidePipe* sp = side_pipe();
    if (!sp) return SLA_ERR_CUDA;
    // fork: the side stream starts after everything already on `s`
    if (cudaEventRecord(sp->fork, s) != cudaSuccess || cudaStreamWaitEvent(sp->side, sp->fork, 0) != cudaSuccess)
      return SLA_ERR_CUDA;
    // kv_prep on fewer CTAs per SM, so that the mask kernels find room beside it
    st_kv = precompute_impl(pl, p, K, V, pw, hz, ws, sp->side, SLA_OVERLAP_KV_CTAS_PER_SM);
    // join (recorded whatever happened, so `s` never waits on a stale event)
    const bool joined = cudaEventRecord(sp->join, sp->side) == cudaSuccess;
    st = predict_mask_impl(pl, p, Q, K, wq, wk, mc, lut, ws, s);
    if (st == SLA_OK) st = pairing_impl(pl, lut, ws, s);
    if (!joined || cudaStreamWaitEvent(s, sp->join, 0) != cudaSuccess) return SLA_ERR_CUDA;
  }
  SLA_TRY(st_kv);
  SLA_TRY(st);
  SLA_TRY(aggregate_impl(pl, mc, hz, ws, s));
  return fused_impl(pl, p, Q, K, V, lut, proj_b, alpha, O, ws, s, nullptr, nullptr, /*pair=*/false);
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
struct BwdLayout {
  size_t err, mm, hagg, drow, dqlin, dhzq, mmt, dhzk, dklin, dvlin, ubuf, rcnt, rptr, rows, pairs, kpairs, pov, end;
};

BwdLayout bwd_layout_of(const Plan& p) {
  BwdLayout L;
  const size_t Tqp = (size_t)((p.Tq + 7) & ~7);
  const size_t act32 = (size_t)p.BH * p.N * p.d * 4;
  size_t o = 0;
  L.err = o;   o = align_up(o + 256);
  L.mm = o;    o = align_up(o + (size_t)p.BH * p.Tq * p.Tkvp * 2);
  L.hagg = o;  o = align_up(o + (size_t)p.BH * p.Tq * p.NN * 2);
  L.drow = o;  o = align_up(o + (size_t)p.BH * p.Tq * 64 * 8);
  L.dqlin = o; o = align_up(o + act32);
  L.dhzq = o;  o = align_up(o + (size_t)p.BH * p.Tq * p.NN * 2);
  L.mmt = o;   o = align_up(o + (size_t)p.BH * p.Tkv * Tqp * 2);
  L.dhzk = o;  o = align_up(o + (size_t)p.BH * p.Tkv * p.NN * 2);
  L.dklin = o; o = align_up(o + act32);
  L.dvlin = o; o = align_up(o + act32);
  L.ubuf = o;  o = align_up(o + (size_t)p.BH * p.Tkv * 64 * p.d * 2);
  L.rcnt = o;  o = align_up(o + (size_t)p.BH * p.Tkv * 4);
  L.rptr = o;  o = align_up(o + (size_t)p.BH * (p.Tkv + 1) * 4);
  L.rows = o;  o = align_up(o + (size_t)p.BH * p.Tq * p.nh * 4);
  L.pairs = o; o = align_up(o + (size_t)p.BH * ((p.Tq + 1) / 2) * 8);
  L.kpairs = o; o = align_up(o + (size_t)p.BH * ((p.Tkv + 1) / 2) * 8);
  L.pov = o;   o = align_up(o + pairing_overlap_bytes(p.BH, std::max(p.Tq, p.Tkv)));
  L.end = o;
  return L;
}

sla_status_t backward_impl(const Plan& pl, const sla_params_t* p, const void* Q, const void* K,
                           const void* V, const int8_t* mc, const int32_t* lut, const void* hz,
                           const float* proj_w, const float* proj_b, const float* alpha,
                           const float* o_sparse, const float* lse, const void* dO, void* dQ,
                           void* dK, void* dV, float* dproj_w, float* dproj_b, float* dalpha,
                           void* ws, cudaStream_t s) {
  const BwdLayout L = bwd_layout_of(pl);
  const bool alpha_mode = p->combine == SLA_COMBINE_ALPHA;
  const int Tqp = (pl.Tq + 7) & ~7;
  int* err = at<int>(ws, L.err);
  // the forward's [H'_i^T | Z_i] (recomputed: the same 0/1 product as the forward)
  __nv_bfloat16* mm = at<__nv_bfloat16>(ws, L.mm);
  __nv_bfloat16* hagg = at<__nv_bfloat16>(ws, L.hagg);
  SLA_TRY(cuda_status(launch_marg_matrix(mc, mm, pl.BH, pl.Tq, pl.Tkv, pl.Tkvp, pl.all, s)));
  SLA_TRY(zero_one_product(pl, mm, pl.Tq, pl.Tkv, pl.Tkvp, hz, hagg, err, s));
  // outputs accumulated with atomics start at zero
  if (dproj_w && !alpha_mode &&
      cudaMemsetAsync(dproj_w, 0, (size_t)pl.d * pl.d * 4, s) != cudaSuccess)
    return SLA_ERR_CUDA;
  if (dproj_b && !alpha_mode && cudaMemsetAsync(dproj_b, 0, (size_t)pl.d * 4, s) != cudaSuccess)
    return SLA_ERR_CUDA;
  if (dalpha && alpha_mode && cudaMemsetAsync(dalpha, 0, (size_t)pl.BH * 4, s) != cudaSuccess)
    return SLA_ERR_CUDA;
  // query side of the linear branch and of the combine
  BwdRowsArgs ra;
  ra.Q = static_cast<const __nv_bfloat16*>(Q);
  ra.os = o_sparse;
  ra.dO = static_cast<const __nv_bfloat16*>(dO);
  for (int i = 0; i < 3; ++i) {
    ra.sq[i] = p->stride_q[i];
    ra.so[i] = p->stride_o[i];
  }
  ra.hagg = hagg;
  ra.alpha = alpha_mode ? alpha : nullptr;
  ra.lse = lse;
  ra.ld2 = at<float2>(ws, L.drow);
  ra.dq_lin = at<float>(ws, L.dqlin);
  ra.dhz = at<__nv_bfloat16>(ws, L.dhzq);
  ra.dalpha = alpha_mode ? dalpha : nullptr;
  ra.dproj_b = alpha_mode ? nullptr : dproj_b;
  ra.H = pl.H;
  ra.N = pl.N;
  ra.Tq = pl.Tq;
  ra.NN = pl.NN;
  ra.combine = p->combine;
  ra.phi = pl.phi;
  ra.eps = p->eps;
  if (pl.d == 128) {
    // tensor-core version: both query blocks of a pair per CTA
    CUtensorMap mh, mz;
    const uint64_t dh[4] = {(uint64_t)pl.d, (uint64_t)pl.d, (uint64_t)pl.Tq, (uint64_t)pl.BH};
    const uint64_t sh[3] = {(uint64_t)pl.d * 2, (uint64_t)pl.NN * 2, (uint64_t)pl.Tq * pl.NN * 2};
    const uint32_t bxh[4] = {64, (uint32_t)pl.d, 1, 1};
    const uint64_t dz[3] = {(uint64_t)pl.NN, (uint64_t)pl.Tq, (uint64_t)pl.BH};
    const uint64_t sz[2] = {(uint64_t)pl.NN * 2, (uint64_t)pl.Tq * pl.NN * 2};
    const uint32_t bxz[3] = {64, 1, 1};
    if (!encode(&mh, hagg, 4, dh, sh, bxh) || !encode(&mz, hagg, 3, dz, sz, bxz, false))
      return SLA_ERR_CUDA;
    BwdRowsArgs rt = ra;
    rt.dproj_b = nullptr;
    SLA_TRY(cuda_status(launch_bwd_rows_tc(mh, mz, rt, err, pl.BH, s)));
    if (!alpha_mode && dproj_b)
      SLA_TRY(cuda_status(launch_colsum(static_cast<const __nv_bfloat16*>(dO), p->stride_o, pl.H,
                                        pl.N, pl.BH, pl.d, dproj_b, s)));
  } else {
    SLA_TRY(cuda_status(launch_bwd_rows(ra, pl.d, pl.BH, s)));
  }
  // dh'_j = sum of dH'_i over the query blocks that have j marginal
  __nv_bfloat16* mmt = at<__nv_bfloat16>(ws, L.mmt);
  SLA_TRY(cuda_status(launch_marg_matrix_t(mc, mmt, pl.BH, pl.Tq, pl.Tkv, Tqp, pl.all, s)));
  SLA_TRY(zero_one_product(pl, mmt, pl.Tkv, pl.Tq, Tqp, ra.dhz, at<__nv_bfloat16>(ws, L.dhzk), err, s));
  // key side of the linear branch
  BwdKeysArgs ka;
  ka.K = static_cast<const __nv_bfloat16*>(K);
  ka.V = static_cast<const __nv_bfloat16*>(V);
  for (int i = 0; i < 3; ++i) {
    ka.sk[i] = p->stride_k[i];
    ka.sv[i] = p->stride_v[i];
  }
  ka.proj_w = alpha_mode ? nullptr : proj_w;
  ka.dhz = at<__nv_bfloat16>(ws, L.dhzk);
  ka.dk_lin = at<float>(ws, L.dklin);
  ka.dv_lin = at<float>(ws, L.dvlin);
  ka.dproj_w = alpha_mode ? nullptr : dproj_w;
  ka.BH = pl.BH;
  ka.H = pl.H;
  ka.N = pl.N;
  ka.Tkv = pl.Tkv;
  ka.NN = pl.NN;
  ka.phi = pl.phi;
  if (pl.d == 128) {
    // tensor-core version: both key blocks of a pair per CTA; dW by a split-K product
    __nv_bfloat16* dhzk = at<__nv_bfloat16>(ws, L.dhzk);
    __nv_bfloat16* ubuf = at<__nv_bfloat16>(ws, L.ubuf);
    CUtensorMap mg, mz, mk2, mv2, mu;
    const uint64_t dg[4] = {(uint64_t)pl.d, (uint64_t)pl.d, (uint64_t)pl.Tkv, (uint64_t)pl.BH};
    const uint64_t sg[3] = {(uint64_t)pl.d * 2, (uint64_t)pl.NN * 2, (uint64_t)pl.Tkv * pl.NN * 2};
    const uint32_t bxg[4] = {64, (uint32_t)pl.d, 1, 1};
    const uint64_t dz[3] = {(uint64_t)pl.NN, (uint64_t)pl.Tkv, (uint64_t)pl.BH};
    const uint64_t sz[2] = {(uint64_t)pl.NN * 2, (uint64_t)pl.Tkv * pl.NN * 2};
    const uint32_t bxz[3] = {64, 1, 1};
    const uint64_t du[3] = {(uint64_t)pl.d, (uint64_t)pl.Tkv * 64, (uint64_t)pl.BH};
    const uint64_t su[2] = {(uint64_t)pl.d * 2, (uint64_t)pl.Tkv * 64 * pl.d * 2};
    const uint32_t bxu[3] = {64, 128, 1};
    if (!encode(&mg, dhzk, 4, dg, sg, bxg) || !encode(&mz, dhzk, 3, dz, sz, bxz, false) ||
        !map_bhnd(&mk2, K, pl, p->stride_k, 128) || !map_bhnd(&mv2, V, pl, p->stride_v, 128) ||
        !encode(&mu, ubuf, 3, du, su, bxu))
      return SLA_ERR_CUDA;
    const bool want_dw = !alpha_mode && proj_w && dproj_w;
    SLA_TRY(cuda_status(launch_bwd_keys_tc(mg, mz, mk2, mv2, ka, want_dw ? ubuf : nullptr, err, s)));
    if (want_dw) SLA_TRY(cuda_status(launch_dw(mu, mv2, pl.H, pl.BH, pl.Tkv, dproj_w, err, s)));
  } else {
    SLA_TRY(cuda_status(launch_bwd_keys(ka, pl.d, s)));
  }
  // sparse branch
  int32_t* rcnt = at<int32_t>(ws, L.rcnt);
  int32_t* rptr = at<int32_t>(ws, L.rptr);
  int32_t* rows = at<int32_t>(ws, L.rows);
  SLA_TRY(cuda_status(launch_rlut(mc, rcnt, rptr, rows, pl.BH, pl.Tq, pl.Tkv, pl.nh, s)));
  // the dQ kernel's query-block pairs (as in the forward) and the dK / dV
  // kernel's key-block pairs (by overlap of the reverse lists)
  int2* pairs = at<int2>(ws, L.pairs);
  int2* kpairs = at<int2>(ws, L.kpairs);
  uint16_t* pov = at<uint16_t>(ws, L.pov);  // used by one pairing at a time (stream order)
  SLA_TRY(cuda_status(launch_pairing(lut, pl.BH, pl.Tq, pl.nh, pl.Tkv, pov, pairs, s)));
  SLA_TRY(cuda_status(launch_pairing_csr(rows, rptr, (int64_t)pl.Tq * pl.nh, pl.BH, pl.Tkv, pl.Tq, pov, kpairs,
                                         s)));
  BwdSparseArgs sa;
  sa.lut = lut;
  sa.rptr = rptr;
  sa.rows = rows;
  sa.ld2 = ra.ld2;
  sa.alpha = alpha_mode ? alpha : nullptr;
  sa.pairs = nullptr;
  sa.err = err;
  sa.H = pl.H;
  sa.N = pl.N;
  sa.Tq = pl.Tq;
  sa.Tkv = pl.Tkv;
  sa.nh = pl.nh;
  sa.combine = p->combine;
  sa.scale = (float)(1.0 / std::sqrt((double)pl.d));
  sa.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)pl.d));
  {
    CUtensorMap mq, mdo, mk, mv;
    if (!map_bhnd(&mq, Q, pl, p->stride_q, 64) || !map_bhnd(&mdo, dO, pl, p->stride_o, 64) ||
        !map_bhnd(&mk, K, pl, p->stride_k, 64) || !map_bhnd(&mv, V, pl, p->stride_v, 64))
      return SLA_ERR_CUDA;
    BwdSparseArgs qa = sa;
    qa.pairs = pairs;
    qa.q_lin = ra.dq_lin;
    qa.v_lin = nullptr;
    qa.out0 = static_cast<__nv_bfloat16*>(dQ);
    qa.out1 = nullptr;
    for (int i = 0; i < 3; ++i) qa.s0[i] = qa.s1[i] = p->stride_q[i];
    SLA_TRY(cuda_status(launch_bwd_dq(mq, mdo, mk, mv, qa, pl.d, pl.BH, s)));
  }
  {
    CUtensorMap mk2, mv2, mq1, mdo1;
    if (!map_bhnd(&mk2, K, pl, p->stride_k, 64) || !map_bhnd(&mv2, V, pl, p->stride_v, 64) ||
        !map_bhnd(&mq1, Q, pl, p->stride_q, 64) || !map_bhnd(&mdo1, dO, pl, p->stride_o, 64))
      return SLA_ERR_CUDA;
    BwdSparseArgs kb = sa;
    kb.pairs = kpairs;
    kb.q_lin = ka.dk_lin;
    kb.v_lin = ka.dv_lin;
    kb.out0 = static_cast<__nv_bfloat16*>(dK);
    kb.out1 = static_cast<__nv_bfloat16*>(dV);
    for (int i = 0; i < 3; ++i) {
      kb.s0[i] = p->stride_k[i];
      kb.s1[i] = p->stride_v[i];
    }
    SLA_TRY(cuda_status(launch_bwd_dkdv(mk2, mv2, mq1, mdo1, kb, pl.d, pl.BH, s)));
  }
  return SLA_OK;
}

// One thread waits on an mbarrier that nothing arrives at: the bounded wait gives
// up after SLA_WAIT_TIMEOUT_NS, records the timeout in the error word and the
// kernel returns (the failure path of every wait in the library, without a fault).
__global__ void selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, err, DEV_TIMEOUT_SYNC);
}

}  // namespace

extern "C" {

void sla_params_default(sla_params_t* p, int B, int H, int N, int d, float k_h, float k_l,
                        int combine) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->B = B;
  p->H = H;
  p->N = N;
  p->d = d;
  p->b_q = 64;
  p->b_kv = 64;
  p->k_h = k_h;
  p->k_l = k_l;
  p->combine = combine;
  p->qk_prec = SLA_QK_BF16;
  p->smooth_k = 0;
  p->eps = 1e-5f;
  p->phi = SLA_PHI_SOFTMAX;
  p->linear_over_all = 0;
  p->pv_prec = SLA_PV_BF16;
  const int64_t s[3] = {(int64_t)H * N * d, (int64_t)N * d, (int64_t)d};
  for (int i = 0; i < 3; ++i) {
    p->stride_q[i] = s[i];
    p->stride_k[i] = s[i];
    p->stride_v[i] = s[i];
    p->stride_o[i] = s[i];
  }
}

sla_status_t sla_block_counts(const sla_params_t* p, int* T_q, int* T_kv, int* n_h, int* n_l) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (T_q) *T_q = pl.Tq;
  if (T_kv) *T_kv = pl.Tkv;
  if (n_h) *n_h = pl.nh;
  if (n_l) *n_l = pl.nl;
  return SLA_OK;
}

sla_status_t sla_workspace_size(const sla_params_t* p, size_t* bytes) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!bytes) return SLA_ERR_INVALID_ARG;
  *bytes = layout_of(pl).end;
  return SLA_OK;
}

sla_status_t sla_hz_size(const sla_params_t* p, size_t* bytes) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!bytes) return SLA_ERR_INVALID_ARG;
  *bytes = (size_t)pl.BH * pl.Tkv * pl.NN * 2;
  return SLA_OK;
}

sla_status_t sla_attention_workspace_size(const sla_params_t* p, size_t* bytes) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!bytes) return SLA_ERR_INVALID_ARG;
  *bytes = layout_of(pl).end_attn;
  return SLA_OK;
}

sla_status_t sla_predict_mask(const sla_params_t* p, const void* Q, const void* K, const float* Wq,
                              const float* Wk, int8_t* mc, int32_t* lut, void* workspace,
                              size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !mc || !lut || !aligned16(Q) || !aligned16(K)) return SLA_ERR_INVALID_ARG;
  if ((Wq && !aligned16(Wq)) || (Wk && !aligned16(Wk))) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return predict_mask_impl(pl, p, Q, K, Wq, Wk, mc, lut, workspace,
                           reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_router_probs(const sla_params_t* p, const void* Q, const void* K, const float* Wq,
                              const float* Wk, float* Pc, void* workspace, size_t workspace_bytes,
                              sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !Pc || !aligned16(Q) || !aligned16(K) || !aligned16(Pc)) return SLA_ERR_INVALID_ARG;
  if ((Wq && !aligned16(Wq)) || (Wk && !aligned16(Wk))) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = layout_of(pl);
  const float *qsrc = nullptr, *ksrc = nullptr;
  SLA_TRY(router_inputs(pl, p, Q, K, Wq, Wk, workspace, s, &qsrc, &ksrc));
  LogitArgs la;
  la.Qc = qsrc;
  la.Kc = ksrc;
  la.keys = at<uint32_t>(workspace, L.keys);
  la.d = pl.d;
  la.Tq = pl.Tq;
  la.Tkv = pl.Tkv;
  SLA_TRY(cuda_status(launch_logits(la, pl.BH, s)));
  return cuda_status(launch_router_probs(la.keys, Pc, pl.Tkv, (int64_t)pl.BH * pl.Tq, s));
}

sla_status_t sla_soft_topk(const sla_params_t* p, const float* Pc, float tau, float* M, float* lambda,
                           sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Pc || !M || !lambda || !aligned16(Pc) || !aligned16(M)) return SLA_ERR_INVALID_ARG;
  // the kernel divides by tau in fp32: tau below the normal range (or whose
  // reciprocal overflows) would turn (P - lambda) / tau into inf * 0 = NaN
  if (!(tau >= 1.1754944e-38f) || !std::isfinite(tau) || !std::isfinite(1.f / tau)) return SLA_ERR_INVALID_ARG;
  return cuda_status(launch_soft_topk(Pc, M, lambda, pl.Tkv, (int64_t)pl.BH * pl.Tq, pl.nh, tau,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

sla_status_t sla_precompute_linear(const sla_params_t* p, const void* K, const void* V,
                                   const float* proj_w, void* hz, void* workspace,
                                   size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!K || !V || !hz || !aligned16(K) || !aligned16(V) || !aligned16(hz)) return SLA_ERR_INVALID_ARG;
  if (proj_w && !aligned16(proj_w)) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return precompute_impl(pl, p, K, V, proj_w, hz, workspace, reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_forward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                         const int8_t* mc, const int32_t* lut, const void* hz,
                         const float* proj_b, const float* alpha, void* O, void* workspace,
                         size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !mc || !lut || !hz || !O) return SLA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(hz))
    return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return forward_impl(pl, p, Q, K, V, mc, lut, hz, proj_b, alpha, O, workspace,
                      reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_forward_train(const sla_params_t* p, const void* Q, const void* K,
                               const void* V, const int8_t* mc, const int32_t* lut,
                               const void* hz, const float* proj_b, const float* alpha, void* O,
                               float* lse, float* o_sparse, void* workspace,
                               size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !mc || !lut || !hz || !O || !lse || !o_sparse) return SLA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(hz) ||
      !aligned16(o_sparse))
    return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return forward_impl(pl, p, Q, K, V, mc, lut, hz, proj_b, alpha, O, workspace,
                      reinterpret_cast<cudaStream_t>(stream), lse, o_sparse);
}

sla_status_t sla_attention(const sla_params_t* p, const void* Q, const void* K, const void* V,
                           const float* proj_w, const float* proj_b, const float* alpha,
                           const float* Wq, const float* Wk, void* O, void* workspace,
                           size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !O) return SLA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_ATTN));
  return attention_impl(pl, p, Q, K, V, proj_w, proj_b, alpha, Wq, Wk, O, workspace,
                        reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_attention_host_workspace_size(const sla_params_t* p, size_t* bytes) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!bytes) return SLA_ERR_INVALID_ARG;
  *bytes = layout_of(pl).end_host;
  return SLA_OK;
}

// Copy streams and events of the host-buffer entry point, created once per device
// (no device memory): chunk c's host-to-device copies run on `h2d`, its compute
// on the caller's stream, its device-to-host copy on `d2h`.
constexpr int kHostChunks = 6;
struct HostPipes {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, end = nullptr, in[kHostChunks] = {}, out[kHostChunks] = {};
  bool ok = false;
};

HostPipes* host_pipes() {
  static std::mutex mu;
  static HostPipes pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  HostPipes& hp = pipes[dev];
  if (!hp.ok) {
    bool good = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&hp.end, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; c < kHostChunks && good; ++c)
      good = cudaEventCreateWithFlags(&hp.in[c], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.out[c], cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    hp.ok = true;
  }
  return &hp;
}

sla_status_t sla_attention_host(const sla_params_t* p, const void* Q_host, const void* K_host,
                                const void* V_host, const float* proj_w, const float* proj_b,
                                const float* alpha, const float* Wq, const float* Wk,
                                void* O_host, void* workspace, size_t workspace_bytes,
                                sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q_host || !K_host || !V_host || !O_host) return SLA_ERR_INVALID_ARG;
  if (!contiguous(p)) return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_HOST));
  const Layout L = layout_of(pl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  HostPipes* hp = host_pipes();
  if (!hp) return SLA_ERR_CUDA;
  uint8_t* dq = at<uint8_t>(workspace, L.hq);
  uint8_t* dk = at<uint8_t>(workspace, L.hk);
  uint8_t* dv = at<uint8_t>(workspace, L.hv);
  uint8_t* dout = at<uint8_t>(workspace, L.ho);
  const uint8_t* qh = static_cast<const uint8_t*>(Q_host);
  const uint8_t* kh = static_cast<const uint8_t*>(K_host);
  const uint8_t* vh = static_cast<const uint8_t*>(V_host);
  uint8_t* oh = static_cast<uint8_t*>(O_host);
  // The (batch, head) problems are independent: chunks of heads are copied in,
  // computed and copied out in a pipeline, so the copies of one chunk overlap the
  // compute of another (the chunks' computations share the workspace one after
  // the other on `stream`).
  const int nchunk = pl.BH < kHostChunks ? pl.BH : kHostChunks;
  const size_t head_bytes = (size_t)pl.N * pl.d * 2;
  SLA_TRY(cuda_status(cudaEventRecord(hp->start, s)));
  SLA_TRY(cuda_status(cudaStreamWaitEvent(hp->h2d, hp->start, 0)));
  SLA_TRY(cuda_status(cudaStreamWaitEvent(hp->d2h, hp->start, 0)));
  for (int c = 0; c < nchunk; ++c) {
    const int b0 = (int)((int64_t)pl.BH * c / nchunk), b1 = (int)((int64_t)pl.BH * (c + 1) / nchunk);
    const size_t off = (size_t)b0 * head_bytes, bytes = (size_t)(b1 - b0) * head_bytes;
    SLA_TRY(cuda_status(cudaMemcpyAsync(dq + off, qh + off, bytes, cudaMemcpyHostToDevice, hp->h2d)));
    SLA_TRY(cuda_status(cudaMemcpyAsync(dk + off, kh + off, bytes, cudaMemcpyHostToDevice, hp->h2d)));
    SLA_TRY(cuda_status(cudaMemcpyAsync(dv + off, vh + off, bytes, cudaMemcpyHostToDevice, hp->h2d)));
    SLA_TRY(cuda_status(cudaEventRecord(hp->in[c], hp->h2d)));
    SLA_TRY(cuda_status(cudaStreamWaitEvent(s, hp->in[c], 0)));
    // the chunk as a problem of its own: B = 1, H = its heads, contiguous
    sla_params_t sp = *p;
    sp.B = 1;
    sp.H = b1 - b0;
    const int64_t st[3] = {(int64_t)sp.H * pl.N * pl.d, (int64_t)pl.N * pl.d, (int64_t)pl.d};
    for (int i = 0; i < 3; ++i) sp.stride_q[i] = sp.stride_k[i] = sp.stride_v[i] = sp.stride_o[i] = st[i];
    Plan sub;
    SLA_TRY(make_plan(&sp, &sub));
    SLA_TRY(attention_impl(sub, &sp, dq + off, dk + off, dv + off, proj_w, proj_b, alpha ? alpha + b0 : nullptr,
                           Wq, Wk, dout + off, workspace, s));
    SLA_TRY(cuda_status(cudaEventRecord(hp->out[c], s)));
    SLA_TRY(cuda_status(cudaStreamWaitEvent(hp->d2h, hp->out[c], 0)));
    SLA_TRY(cuda_status(cudaMemcpyAsync(oh + off, dout + off, bytes, cudaMemcpyDeviceToHost, hp->d2h)));
  }
  SLA_TRY(cuda_status(cudaEventRecord(hp->end, hp->d2h)));
  return cuda_status(cudaStreamWaitEvent(s, hp->end, 0));
}

sla_status_t sla_aggregate_marginal(const sla_params_t* p, const int8_t* mc, const void* hz,
                                    void* workspace, size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!mc || !hz || !aligned16(hz)) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return aggregate_impl(pl, mc, hz, workspace, reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_fused_forward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                               const int32_t* lut, const float* proj_b, const float* alpha,
                               void* O, void* workspace, size_t workspace_bytes,
                               sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !lut || !O) return SLA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return fused_impl(pl, p, Q, K, V, lut, proj_b, alpha, O, workspace,
                    reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_pair_query_blocks(const sla_params_t* p, const int32_t* lut, void* workspace,
                                   size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!lut) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return pairing_impl(pl, lut, workspace, reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_fused_forward_paired(const sla_params_t* p, const void* Q, const void* K, const void* V,
                                      const int32_t* lut, const float* proj_b, const float* alpha,
                                      void* O, void* workspace, size_t workspace_bytes,
                                      sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !lut || !O) return SLA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  SLA_TRY(check_ws(pl, workspace, workspace_bytes, WS_BASE));
  return fused_impl(pl, p, Q, K, V, lut, proj_b, alpha, O, workspace,
                    reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, false);
}

sla_status_t sla_workspace_pairs(const sla_params_t* p, size_t* offset, size_t* count) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!offset || !count) return SLA_ERR_INVALID_ARG;
  *offset = layout_of(pl).pairs;
  *count = (size_t)pl.BH * ((pl.Tq + 1) / 2);
  return SLA_OK;
}

sla_status_t sla_backward_workspace_size(const sla_params_t* p, size_t* bytes) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!bytes) return SLA_ERR_INVALID_ARG;
  *bytes = bwd_layout_of(pl).end;
  return SLA_OK;
}

sla_status_t sla_backward(const sla_params_t* p, const void* Q, const void* K, const void* V,
                          const int8_t* mc, const int32_t* lut, const void* hz,
                          const float* proj_w, const float* proj_b, const float* alpha,
                          const float* o_sparse, const float* lse, const void* dO, void* dQ,
                          void* dK, void* dV, float* dproj_w, float* dproj_b, float* dalpha,
                          void* workspace, size_t workspace_bytes, sla_stream_t stream) {
  Plan pl;
  SLA_TRY(make_plan(p, &pl));
  if (!Q || !K || !V || !mc || !lut || !hz || !o_sparse || !lse || !dO || !dQ || !dK || !dV)
    return SLA_ERR_INVALID_ARG;
  for (const void* x : {Q, K, V, (const void*)o_sparse, dO, (const void*)dQ, (const void*)dK,
                        (const void*)dV, hz})
    if (!aligned16(x)) return SLA_ERR_INVALID_ARG;
  if (p->combine == SLA_COMBINE_ALPHA && !alpha) return SLA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      workspace_bytes < bwd_layout_of(pl).end)
    return SLA_ERR_WORKSPACE;
  return backward_impl(pl, p, Q, K, V, mc, lut, hz, proj_w, proj_b, alpha, o_sparse, lse, dO, dQ, dK, dV,
                       dproj_w, dproj_b, dalpha, workspace, reinterpret_cast<cudaStream_t>(stream));
}

sla_status_t sla_selftest_wait_timeout(void* workspace, sla_stream_t stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return SLA_ERR_WORKSPACE;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<int*>(workspace));
  return cuda_status(cudaGetLastError());
}

sla_status_t sla_get_device_status(void* workspace, sla_stream_t stream, int* detail) {
  if (!workspace) return SLA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int code = 0;
  if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SLA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SLA_ERR_CUDA;
  if (code != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return SLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SLA_ERR_CUDA;
  }
  if (detail) *detail = code;
  if (code == DEV_OK) return SLA_OK;
  if (code == DEV_BAD_INDEX) return SLA_ERR_DEVICE_BAD_INDEX;
  return SLA_ERR_DEVICE_TIMEOUT;
}

const char* sla_status_string(sla_status_t s) {
  switch (s) {
    case SLA_OK: return "SLA_OK";
    case SLA_ERR_INVALID_ARG: return "SLA_ERR_INVALID_ARG";
    case SLA_ERR_UNSUPPORTED: return "SLA_ERR_UNSUPPORTED";
    case SLA_ERR_WORKSPACE: return "SLA_ERR_WORKSPACE";
    case SLA_ERR_CUDA: return "SLA_ERR_CUDA";
    case SLA_ERR_DEVICE_TIMEOUT: return "SLA_ERR_DEVICE_TIMEOUT";
    case SLA_ERR_DEVICE_BAD_INDEX: return "SLA_ERR_DEVICE_BAD_INDEX";
  }
  return "SLA_ERR_UNKNOWN";
}

int sla_abi_version(void) { return 104; }

}  // extern "C"
