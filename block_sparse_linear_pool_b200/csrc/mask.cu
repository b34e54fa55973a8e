// Compressed mask prediction ("SLA: Beyond Sparsity in Diffusion Transformers
// via Fine-Tunable Sparse-Linear Attention", §2 Q2 steps 1-2 and Fig. 4 left;
// "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §4):
//   pool_kernel     mean of Q and K over 64-token blocks (real tokens only)
//   kmean_kernel    token mean of K per head (smooth-K, SLA §7 item 3)
//   router_kernel   x <- (x - mean) W^T for the SLA2 router projections
//   select_kernel   logits = Q_c K_c^T / sqrt(d) for 8 query blocks per CTA,
//                   then an exact row-wise top-n_h / bottom-n_l selection by
//                   radix search over order-preserving 32-bit keys.
#include "kernels.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// pool: one warp per 64-token block; lane l sums columns [l*CPL, (l+1)*CPL).
// grid (ceil(T/8), B*H, 2): z = 0 pools Q into Qc, z = 1 pools K into Kc.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(PoolArgs a) {
  constexpr int CPL = D / 32;  // columns per lane: 4 (d=128) or 2 (d=64)
  const int w = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int blk = blockIdx.x * 8 + w;
  const int bh = blockIdx.y;
  const int T = a.T;
  if (blk >= T) return;
  const int b = bh / a.H, h = bh % a.H;
  const __nv_bfloat16* src = blockIdx.z == 0 ? a.Q : a.K;
  const int64_t* st = blockIdx.z == 0 ? a.sq : a.sk;
  float* dst = blockIdx.z == 0 ? a.Qc : a.Kc;
  const __nv_bfloat16* base = src + (int64_t)b * st[0] + (int64_t)h * st[1];
  const int t0 = blk * a.bs;
  const int cnt = min(a.bs, a.N - t0);
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
#pragma unroll 8
  for (int t = 0; t < cnt; ++t) {
    const __nv_bfloat16* row = base + (int64_t)(t0 + t) * st[2] + ln * CPL;
    if constexpr (CPL == 4) {
      uint2 v = __ldg(reinterpret_cast<const uint2*>(row));
      __nv_bfloat162 p0 = *reinterpret_cast<__nv_bfloat162*>(&v.x);
      __nv_bfloat162 p1 = *reinterpret_cast<__nv_bfloat162*>(&v.y);
      acc[0] += __low2float(p0); acc[1] += __high2float(p0);
      acc[2] += __low2float(p1); acc[3] += __high2float(p1);
    } else {
      uint32_t v = __ldg(reinterpret_cast<const unsigned int*>(row));
      __nv_bfloat162 p0 = *reinterpret_cast<__nv_bfloat162*>(&v);
      acc[0] += __low2float(p0); acc[1] += __high2float(p0);
    }
  }
  const float inv = 1.f / (float)cnt;
  float* out = dst + ((int64_t)bh * T + blk) * D + ln * CPL;
#pragma unroll
  for (int c = 0; c < CPL; ++c) out[c] = acc[c] * inv;
}

// ---------------------------------------------------------------------------
// kmean: per head, mean over all N tokens of K = sum_j cnt_j Kc_j / N.
// grid (B*H), block D threads.
// ---------------------------------------------------------------------------
__global__ void kmean_kernel(const float* Kc, float* kmean, int T, int N, int bs, int D) {
  const int bh = blockIdx.x, c = threadIdx.x;
  if (c >= D) return;
  double s = 0.0;
  for (int j = 0; j < T; ++j) {
    const int cnt = min(bs, N - j * bs);
    s += (double)Kc[((int64_t)bh * T + j) * D + c] * cnt;
  }
  kmean[(int64_t)bh * D + c] = (float)(s / N);
}

// ---------------------------------------------------------------------------
// router: out[r] = (in[r] - mean) W^T  (W fp32 [D][D], nn.Linear convention,
// identity when W == nullptr).  grid (T, B*H), block D threads.
// ---------------------------------------------------------------------------
__global__ void router_kernel(const float* in, const float* mean, const float* W, float* out,
                              int T, int D) {
  extern __shared__ float xs[];
  const int r = blockIdx.x, bh = blockIdx.y, o = threadIdx.x;
  const float* x = in + ((int64_t)bh * T + r) * D;
  xs[o] = x[o] - (mean ? mean[(int64_t)bh * D + o] : 0.f);
  __syncthreads();
  float acc;
  if (W) {
    acc = 0.f;
    const float* wr = W + (int64_t)o * D;
    for (int k = 0; k < D; ++k) acc = fmaf(xs[k], __ldg(wr + k), acc);
  } else {
    acc = xs[o];
  }
  out[((int64_t)bh * T + r) * D + o] = acc;
}

// ---------------------------------------------------------------------------
// select: 8 query rows per CTA (one warp each), logits for all T_kv key blocks
// kept in shared memory, then row-wise selection.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Among `T` keys in smem, finds the k-th largest key (1 <= k <= T) by a
// most-significant-bit-first radix search.  Returns the key value in *kth and
// the number of elements equal to it that belong to the top k (lowest block
// index first) in *need.
__device__ void kth_largest(const uint32_t* keys, int T, int k, uint32_t* kth, int* need) {
  const int ln = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t mb = mask | (1u << bit);
    const uint32_t cand = prefix | (1u << bit);
    int cnt = 0;
    for (int j = ln; j < T; j += 32) cnt += ((keys[j] & mb) == cand);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= remaining) {
      prefix = cand;
    } else {
      remaining -= cnt;
    }
    mask = mb;
  }
  *kth = prefix;
  *need = remaining;
}

__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int D = a.d;
  const int Tq = a.Tq, Tk = a.Tkv;
  const int bh = blockIdx.y;
  const int w = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int row0 = blockIdx.x * 8;
  float* qs = reinterpret_cast<float*>(sm);                  // [8][D]
  float* kt = qs + 8 * D;                                    // [D][33] transposed chunk
  uint32_t* keys = reinterpret_cast<uint32_t*>(kt + D * 33); // [8][Tk]
  const float* Qc = a.Qc + (int64_t)bh * Tq * D;
  const float* Kc = a.Kc + (int64_t)bh * Tk * D;
  for (int e = threadIdx.x; e < 8 * D; e += 256) {
    const int r = e / D, c = e % D;
    qs[e] = (row0 + r < Tq) ? Qc[(int64_t)(row0 + r) * D + c] : 0.f;
  }
  const float scale = rsqrtf((float)D);
  for (int j0 = 0; j0 < Tk; j0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * D; e += 256) {
      const int jj = e / D, c = e % D;
      kt[c * 33 + jj] = (j0 + jj < Tk) ? Kc[(int64_t)(j0 + jj) * D + c] : 0.f;
    }
    __syncthreads();
    const float* q = qs + w * D;
    float acc = 0.f;
    for (int c = 0; c < D; ++c) acc = fmaf(q[c], kt[c * 33 + ln], acc);
    if (j0 + ln < Tk) keys[w * Tk + j0 + ln] = order_key(acc * scale);
  }
  __syncthreads();
  const int i = row0 + w;
  if (i >= Tq) return;
  const uint32_t* rk = keys + w * Tk;
  // critical: top n_h; kept (critical or marginal): top T_kv - n_l
  uint32_t kh, kk;
  int need_h, need_k;
  kth_largest(rk, Tk, a.nh, &kh, &need_h);
  const int nkeep = Tk - a.nl;
  kth_largest(rk, Tk, nkeep, &kk, &need_k);
  int8_t* mrow = a.mc + ((int64_t)bh * Tq + i) * Tk;
  int32_t* lrow = a.lut + ((int64_t)bh * Tq + i) * a.nh;
  int eq_h = 0, eq_k = 0, ncrit = 0;
  const uint32_t lt = (1u << ln) - 1u;
  for (int j0 = 0; j0 < Tk; j0 += 32) {
    const int j = j0 + ln;
    const bool valid = j < Tk;
    const uint32_t key = valid ? rk[j] : 0u;
    const uint32_t bh_eq = __ballot_sync(0xffffffffu, valid && key == kh);
    const uint32_t bk_eq = __ballot_sync(0xffffffffu, valid && key == kk);
    const bool crit = valid && (key > kh || (key == kh && eq_h + __popc(bh_eq & lt) < need_h));
    const bool keep = valid && (key > kk || (key == kk && eq_k + __popc(bk_eq & lt) < need_k));
    eq_h += __popc(bh_eq);
    eq_k += __popc(bk_eq);
    const uint32_t bc = __ballot_sync(0xffffffffu, crit);
    if (valid) mrow[j] = crit ? (int8_t)1 : (keep ? (int8_t)0 : (int8_t)-1);
    if (crit) lrow[ncrit + __popc(bc & lt)] = j;
    ncrit += __popc(bc);
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_pool(const PoolArgs& a, int D, int BH, cudaStream_t s) {
  dim3 grid((a.T + 7) / 8, BH, 2);
  if (D == 128) pool_kernel<128><<<grid, 256, 0, s>>>(a);
  else pool_kernel<64><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router(const float* Qc, const float* Kc, float* Qr, float* Kr, float* kmean,
                          const float* Wq, const float* Wk, bool smooth, int BH, int Tq, int Tk,
                          int N, int bs, int D, cudaStream_t s) {
  if (smooth) kmean_kernel<<<BH, D, 0, s>>>(Kc, kmean, Tk, N, bs, D);
  router_kernel<<<dim3(Tq, BH), D, D * sizeof(float), s>>>(Qc, nullptr, Wq, Qr, Tq, D);
  router_kernel<<<dim3(Tk, BH), D, D * sizeof(float), s>>>(Kc, smooth ? kmean : nullptr, Wk, Kr,
                                                          Tk, D);
  return cudaGetLastError();
}

size_t select_smem_bytes(int D, int Tk) {
  return (size_t)(8 * D + D * 33) * sizeof(float) + (size_t)8 * Tk * sizeof(uint32_t);
}

cudaError_t launch_select(const SelectArgs& a, int BH, cudaStream_t s) {
  const size_t smem = select_smem_bytes(a.d, a.Tkv);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<<<dim3((a.Tq + 7) / 8, BH), 256, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sla
