// Router probabilities and SoftTop-k ("SLA2: Sparse-Linear Attention with
// Learnable Routing and QAT", §4 Learnable Router: P_c from the pooled and
// projected Q, K, row-wise Top-k; §6 Training with SLA2: SoftTop-k, a sigmoid
// with temperature tau and a per-row threshold lambda_i found by binary search
// so that each row keeps the Top-k row sum).
//
//   router_probs_kernel  the logits' order-preserving keys (written by
//                        logits_kernel) back to fp32 s_ij, then
//                        P_c[i][j] = exp(s_ij - max_j s) / sum; one warp per row
//   soft_topk_kernel     per row, lambda_i by bisection on
//                        f(lambda) = sum_j sigmoid((P_ij - lambda) / tau) = n_h
//                        over [min P - 50 tau, max P + 50 tau] (f falls from
//                        ~T to ~0 there), a fixed 40 halvings (fp32 resolution),
//                        then M_ij = sigmoid((P_ij - lambda_i) / tau); one warp
//                        per row, the row staged in shared memory.  The warp's
//                        butterfly sums leave every lane the same f, so the
//                        bisection's branch is warp-uniform.
#include "kernels.cuh"

namespace sla {

namespace {
constexpr int PWARPS = 8;   // rows per CTA, router_probs_kernel
constexpr int SWARPS = 4;   // rows per CTA, soft_topk_kernel
constexpr int ITERS = 40;
constexpr unsigned FULL = 0xffffffffu;

// inverse of the order-preserving key: sign bit set = a non-negative float
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + expf(-x)); }
}  // namespace

__global__ void __launch_bounds__(32 * PWARPS) router_probs_kernel(const uint32_t* __restrict__ keys,
                                                                   float* __restrict__ Pc, int Tkv,
                                                                   int64_t rows) {
  const int64_t r = (int64_t)blockIdx.x * PWARPS + (threadIdx.x >> 5);
  const int ln = threadIdx.x & 31;
  if (r >= rows) return;  // the whole warp
  const uint32_t* kr = keys + r * Tkv;
  float m = -INFINITY;
  for (int j = ln; j < Tkv; j += 32) m = fmaxf(m, key_to_float(kr[j]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  float s = 0.f;
  for (int j = ln; j < Tkv; j += 32) s += expf(key_to_float(kr[j]) - m);
  const float inv = 1.f / warp_sum(s);
  float* pr = Pc + r * Tkv;
  for (int j = ln; j < Tkv; j += 32) pr[j] = expf(key_to_float(kr[j]) - m) * inv;
}

__global__ void __launch_bounds__(32 * SWARPS) soft_topk_kernel(const float* __restrict__ Pc,
                                                                float* __restrict__ M,
                                                                float* __restrict__ lam, int Tkv,
                                                                int64_t rows, float target, float tau) {
  extern __shared__ float srow[];  // [SWARPS][Tkv]
  const int wl = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * SWARPS + wl;
  if (r >= rows) return;  // the whole warp; no block-wide barrier follows
  float* row = srow + (size_t)wl * Tkv;
  const float* pr = Pc + r * Tkv;
  float mn = INFINITY, mx = -INFINITY;
  for (int j = ln; j < Tkv; j += 32) {
    const float v = pr[j];
    row[j] = v;
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
  }
  __syncwarp();
  const float itau = 1.f / tau;
  float lo = mn - 50.f * tau, hi = mx + 50.f * tau;
  for (int it = 0; it < ITERS; ++it) {
    const float mid = 0.5f * (lo + hi);
    float f = 0.f;
    for (int j = ln; j < Tkv; j += 32) f += sigmoid((row[j] - mid) * itau);
    if (warp_sum(f) > target) lo = mid;
    else hi = mid;
  }
  const float l = 0.5f * (lo + hi);
  float* mr = M + r * Tkv;
  for (int j = ln; j < Tkv; j += 32) mr[j] = sigmoid((row[j] - l) * itau);
  if (ln == 0) lam[r] = l;
}

cudaError_t launch_router_probs(const uint32_t* keys, float* Pc, int Tkv, int64_t rows, cudaStream_t s) {
  router_probs_kernel<<<(unsigned)((rows + PWARPS - 1) / PWARPS), 32 * PWARPS, 0, s>>>(keys, Pc, Tkv, rows);
  return cudaGetLastError();
}

cudaError_t launch_soft_topk(const float* Pc, float* M, float* lam, int Tkv, int64_t rows, int nh, float tau,
                             cudaStream_t s) {
  const size_t smem = (size_t)SWARPS * Tkv * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(soft_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  soft_topk_kernel<<<(unsigned)((rows + SWARPS - 1) / SWARPS), 32 * SWARPS, smem, s>>>(Pc, M, lam, Tkv, rows,
                                                                                       (float)nh, tau);
  return cudaGetLastError();
}

}  // namespace sla
