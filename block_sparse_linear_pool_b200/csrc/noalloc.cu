// Mask prediction without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// forward: code running inside a host callback or another library's
// allocation-free hot loop, embedders whose memory is fully pre-planned by an
// arena they do not control, or runtimes that forbid allocation after start-up.
// For them this file keeps the scratch that mask prediction needs (the error
// word, the pooled / routed Q and K blocks and the logit keys) in one
// statically sized device array, so sla_predict_mask_noalloc needs only the
// caller's inputs and outputs.
//
// The array lives for as long as the library is loaded, on every GPU the
// library is used on.  Its device address is looked up once per device (on the
// first call made with that device current) with cudaGetSymbolAddress; that
// first call should therefore happen before any stream capture.  All calls on a
// device share the array and it keeps the last call's contents: calls whose
// executions overlap on the GPU (different streams, or concurrent host
// threads) race on it and must be serialised by the caller.
#include <mutex>

#include "sla.h"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = SLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

void* g_scratch_ptr[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of g_scratch on the current device (looked up once).
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_scratch_once[dev], [dev] {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_scratch);
    g_scratch_ptr[dev] = p;
  });
  if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" sla_status_t sla_predict_mask_noalloc(const sla_params_t* p, const void* Q,
                                                  const void* K, const float* Wq,
                                                  const float* Wk, int8_t* mc, int32_t* lut,
                                                  sla_stream_t stream) {
  int Tq = 0, Tkv = 0, nh = 0, nl = 0;
  sla_status_t st = sla_block_counts(p, &Tq, &Tkv, &nh, &nl);  // validates p
  if (st != SLA_OK) return st;
  if (!Q || !K || !mc || !lut) return SLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) & 15u)
    return SLA_ERR_INVALID_ARG;
  if ((Wq && (reinterpret_cast<uintptr_t>(Wq) & 15u)) || (Wk && (reinterpret_cast<uintptr_t>(Wk) & 15u)))
    return SLA_ERR_INVALID_ARG;
  const int BH = p->B * p->H, d = p->d;
  const bool route = Wq || Wk || p->smooth_k;
  // scratch: error word | logit keys | Q_c | K_c | (routed Q_c | routed K_c | token mean of K)
  const size_t off_keys = 256;
  const size_t off_qc = off_keys + up256((size_t)BH * Tq * Tkv * 4);
  const size_t off_kc = off_qc + up256((size_t)BH * Tq * d * 4);
  const size_t off_qr = off_kc + up256((size_t)BH * Tkv * d * 4);
  const size_t off_kr = off_qr + (route ? up256((size_t)BH * Tq * d * 4) : 0);
  const size_t off_km = off_kr + (route ? up256((size_t)BH * Tkv * d * 4) : 0);
  const size_t need = off_km + (route ? up256((size_t)BH * d * 4) : 0);
  if (need > kScratchBytes) return SLA_ERR_WORKSPACE;  // problem too large for the static scratch

  void* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return SLA_ERR_CUDA;
  unsigned char* s = static_cast<unsigned char*>(base);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the error word must start at zero; everything else is overwritten
  if (cudaMemsetAsync(s, 0, 256, cs) != cudaSuccess) return SLA_ERR_CUDA;

  sla::PoolArgs pa;
  pa.Q = static_cast<const __nv_bfloat16*>(Q);
  pa.K = static_cast<const __nv_bfloat16*>(K);
  for (int i = 0; i < 3; ++i) {
    pa.sq[i] = p->stride_q[i];
    pa.sk[i] = p->stride_k[i];
  }
  pa.Qc = reinterpret_cast<float*>(s + off_qc);
  pa.Kc = reinterpret_cast<float*>(s + off_kc);
  pa.H = p->H;
  pa.N = p->N;
  pa.T = Tq;
  pa.bs = 64;
  if (sla::launch_pool(pa, d, BH, cs) != cudaSuccess) return SLA_ERR_CUDA;
  const float* qsrc = pa.Qc;
  const float* ksrc = pa.Kc;
  if (route) {
    float* qr = reinterpret_cast<float*>(s + off_qr);
    float* kr = reinterpret_cast<float*>(s + off_kr);
    float* km = reinterpret_cast<float*>(s + off_km);
    if (sla::launch_router(pa.Qc, pa.Kc, qr, kr, km, Wq, Wk, p->smooth_k != 0, BH, Tq, Tkv, p->N,
                           64, d, cs) != cudaSuccess)
      return SLA_ERR_CUDA;
    qsrc = qr;
    ksrc = kr;
  }
  sla::SelectArgs sa;
  sa.Qc = qsrc;
  sa.Kc = ksrc;
  sa.keys = reinterpret_cast<uint32_t*>(s + off_keys);
  sa.mc = mc;
  sa.lut = lut;
  sa.d = d;
  sa.Tq = Tq;
  sa.Tkv = Tkv;
  sa.nh = nh;
  sa.nl = nl;
  return sla::launch_select(sa, BH, cs) == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}
