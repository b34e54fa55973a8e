// Low-bit Q and K for the sparse branch ("SLA2: Sparse-Linear Attention with
// Learnable Routing and QAT", §5: Q and K are mapped to FP8 with scales before
// Q K^T, and the product is rescaled).
//
// One scale per (head, 64-row block): s = max|x| / R with R = 448 (the largest
// finite E4M3 value) or 127 (symmetric INT8, the other low-bit format the page
// names); the code is the round-to-nearest-even of x * (R / max|x|) (E4M3 with
// saturation; INT8 clamped to [-127, 127]).  Rows past N in the last block are
// written as zeros, so every block occupies 64 rows.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace sla {

// grid (T, B*H, 2): z = 0 quantises Q, z = 1 quantises K.  128 threads; thread
// t owns row t/2 and the 64 columns starting at 64*(t%2) (d = 128).
__global__ void __launch_bounds__(128) quant_fp8_kernel(QuantArgs a) {
  __shared__ float red[4];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int T = which == 0 ? a.Tq : a.Tkv;
  if (blk >= T) return;
  const int b = bh / a.H, h = bh % a.H;
  const __nv_bfloat16* src = which == 0 ? a.Q : a.K;
  const int64_t* st = which == 0 ? a.sq : a.sk;
  uint8_t* dst = which == 0 ? a.Q8 : a.K8;
  float* scale = which == 0 ? a.scale_q : a.scale_k;
  const int t = threadIdx.x, row = t >> 1, c0 = 64 * (t & 1);
  const int n = 64 * blk + row;
  const bool valid = n < a.N;
  float x[64];
  float amax = 0.f;
  const __nv_bfloat16* p = src + (int64_t)b * st[0] + (int64_t)h * st[1] + (int64_t)n * st[2] + c0;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    uint4 q = valid ? __ldg(reinterpret_cast<const uint4*>(p) + v) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[8 * v + 2 * u] = __low2float(p2[u]);
      x[8 * v + 2 * u + 1] = __high2float(p2[u]);
      amax = fmaxf(amax, fmaxf(fabsf(x[8 * v + 2 * u]), fabsf(x[8 * v + 2 * u + 1])));
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float R = a.int8 ? 127.f : 448.f;
  const float s = amax > 0.f ? amax / R : 1.f;
  const float inv = amax > 0.f ? R / amax : 0.f;
  uint8_t* out = dst + ((int64_t)bh * T * 64 + 64 * blk + row) * 128 + c0;
  if (a.int8) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint32_t w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = min(max(__float2int_rn(x[16 * v + 4 * u + b] * inv), -127), 127);
          word |= (uint32_t)(c & 0xff) << (8 * b);
        }
        w[u] = word;
      }
      reinterpret_cast<uint4*>(out)[v] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (t == 0) scale[(int64_t)bh * T + blk] = s;
    return;
  }
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 16 * v + 4 * u;
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(x[e] * inv, x[e + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(x[e + 2] * inv, x[e + 3] * inv), __NV_SATFINITE, __NV_E4M3);
      w[u] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    reinterpret_cast<uint4*>(out)[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (t == 0) scale[(int64_t)bh * T + blk] = s;
}

// ---------------------------------------------------------------------------
// V for the FP8 P V product: one scale per (head, channel), s_V[c] = max_t |V[t][c]|
// / 448, so that the scale factors out of the sum over keys.  V^ is written
// transposed per 64-token block, [BH][T][d rows][128 B] with the 64 tokens in the
// first 64 bytes of each row (the rest zero): the K-major B operand of the
// kind::f8f6f4 MMA O += P^ V^ (K = tokens).
// ---------------------------------------------------------------------------
// grid (ceil(N / 256), B*H), d threads: per-channel |V| maximum into vmax (zeroed
// by the caller; non-negative floats order like their bit patterns).
__global__ void vamax_kernel(const __nv_bfloat16* __restrict__ V, int64_t s0, int64_t s1, int64_t s2, int H,
                             int N, unsigned int* __restrict__ vmax) {
  const int c = threadIdx.x, bh = blockIdx.y;
  const int n0 = blockIdx.x * 256;
  const __nv_bfloat16* base = V + (int64_t)(bh / H) * s0 + (int64_t)(bh % H) * s1 + c;
  float m = 0.f;
  for (int n = n0; n < min(n0 + 256, N); ++n) m = fmaxf(m, fabsf(__bfloat162float(base[(int64_t)n * s2])));
  atomicMax(vmax + (int64_t)bh * blockDim.x + c, __float_as_uint(m));
}

// grid (T, B*H), d threads: thread c writes row c of block j: 64 E4M3 values of
// V[64 j + t][c] / s_V[c], then 64 zero bytes.
__global__ void vquant_t_kernel(const __nv_bfloat16* __restrict__ V, int64_t s0, int64_t s1, int64_t s2,
                                int H, int N, int T, const unsigned int* __restrict__ vmax,
                                uint8_t* __restrict__ V8T) {
  const int c = threadIdx.x, j = blockIdx.x, bh = blockIdx.y;
  const float amax = __uint_as_float(vmax[(int64_t)bh * blockDim.x + c]);
  const float inv = amax > 0.f ? 448.f / amax : 0.f;
  const __nv_bfloat16* base = V + (int64_t)(bh / H) * s0 + (int64_t)(bh % H) * s1 + c;
  uint8_t* out = V8T + (((int64_t)bh * T + j) * blockDim.x + c) * 128;
#pragma unroll 4
  for (int t = 0; t < 64; t += 4) {
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = 64 * j + t + e;
      x[e] = n < N ? __bfloat162float(base[(int64_t)n * s2]) * inv : 0.f;
    }
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[0], x[1]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x[2], x[3]), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(out + t) = (uint32_t)lo | ((uint32_t)hi << 16);
  }
#pragma unroll
  for (int t = 64; t < 128; t += 16) *reinterpret_cast<uint4*>(out + t) = make_uint4(0, 0, 0, 0);
}

cudaError_t launch_vquant_fp8(const __nv_bfloat16* V, const int64_t* sv, int H, int N, int T, int BH, int D,
                              unsigned int* vmax, uint8_t* V8T, cudaStream_t s) {
  if (cudaMemsetAsync(vmax, 0, (size_t)BH * D * 4, s) != cudaSuccess) return cudaGetLastError();
  vamax_kernel<<<dim3((N + 255) / 256, BH), D, 0, s>>>(V, sv[0], sv[1], sv[2], H, N, vmax);
  vquant_t_kernel<<<dim3(T, BH), D, 0, s>>>(V, sv[0], sv[1], sv[2], H, N, T, vmax, V8T);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const QuantArgs& a, int BH, cudaStream_t s) {
  const int T = a.Tq > a.Tkv ? a.Tq : a.Tkv;
  quant_fp8_kernel<<<dim3(T, BH, 2), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sla
