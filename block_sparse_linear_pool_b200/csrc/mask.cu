// Compressed mask prediction ("SLA: Beyond Sparsity in Diffusion Transformers
// via Fine-Tunable Sparse-Linear Attention", §2 Q2 steps 1-2 and Fig. 4 left;
// "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §4):
//   pool_kernel     mean of Q and K over 64-token blocks (real tokens only)
//   kmean_kernel    token mean of K per head (smooth-K, SLA §7 item 3)
//   router_kernel   x <- (x - mean) W^T for the SLA2 router projections (fp32)
//   select_kernel   logits = Q_c K_c^T / sqrt(d) in fp32 for 8-32 query blocks
//                   per CTA, then an exact row-wise top-n_h / bottom-n_l
//                   selection by radix search over order-preserving 32-bit keys.
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
// router: out[r] = (in[r] - mean) W^T  (W fp32 [D][D], nn.Linear convention;
// identity when W == nullptr).  fp32 tiles: 64 rows x D outputs per CTA, W^T
// and the row tile staged in shared memory; thread (ty, tx) owns rows
// 4ty..4ty+3 and columns tx + 16c.  grid (ceil(T/64), B*H).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ in,
                                                     const float* __restrict__ mean,
                                                     const float* __restrict__ W,
                                                     float* __restrict__ out, int T) {
  extern __shared__ __align__(16) float rsm[];
  constexpr int XS = 68;          // padded row-tile stride (64 rows + 4)
  constexpr int WS = D + 1;       // padded W^T stride
  float* xt = rsm;                // [D][XS]  x^T
  float* wt = rsm + D * XS;       // [D][WS]  W^T
  const int bh = blockIdx.y, r0 = blockIdx.x * 64, tid = threadIdx.x;
  const float* x = in + (int64_t)bh * T * D;
  const float* mu = mean ? mean + (int64_t)bh * D : nullptr;
  for (int e = tid; e < 64 * D; e += 256) {
    const int r = e / D, c = e % D;
    xt[c * XS + r] = (r0 + r < T) ? x[(int64_t)(r0 + r) * D + c] - (mu ? mu[c] : 0.f) : 0.f;
  }
  if (W) {
    for (int e = tid; e < D * D; e += 256) wt[(e % D) * WS + e / D] = __ldg(W + e);
  }
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15;
  float* o = out + (int64_t)bh * T * D;
  if (!W) {
    for (int e = tid; e < 64 * D; e += 256) {
      const int r = e / D, c = e % D;
      if (r0 + r < T) o[(int64_t)(r0 + r) * D + c] = xt[c * XS + r];
    }
    return;
  }
  constexpr int NC = D / 16;
  float acc[4][NC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[i][c] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    const float4 xv = *reinterpret_cast<const float4*>(xt + k * XS + 4 * ty);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float wv = wt[k * WS + tx + 16 * c];
      acc[0][c] = fmaf(xv.x, wv, acc[0][c]);
      acc[1][c] = fmaf(xv.y, wv, acc[1][c]);
      acc[2][c] = fmaf(xv.z, wv, acc[2][c]);
      acc[3][c] = fmaf(xv.w, wv, acc[3][c]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + 4 * ty + i;
    if (r < T) {
#pragma unroll
      for (int c = 0; c < NC; ++c) o[(int64_t)r * D + tx + 16 * c] = acc[i][c];
    }
  }
}

// ---------------------------------------------------------------------------
// select: R query rows per CTA.  Their logits against all T_kv key blocks are
// formed in fp32 (register-blocked: thread (ty, tx) owns rows ty (+16) and
// columns tx + 16c of each 64-column chunk of K_c staged transposed in shared
// memory) and kept as order-preserving keys in shared memory; each warp then
// selects its rows by an exact radix search.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Among `T` keys in shared memory, finds the k-th largest key (1 <= k <= T) by a
// most-significant-digit-first radix search with 8-bit digits (one 256-bin
// histogram per warp).  Returns the key in *kth and the number of elements equal
// to it that belong to the top k (lowest block index first) in *need.
__device__ void kth_largest(const uint32_t* keys, int T, int k, uint32_t* hist, uint32_t* kth,
                            int* need) {
  const int ln = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = ln; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = ln; j < T; j += 32) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending)
    int c[8], lsum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = (int)hist[255 - 8 * ln - i];
      lsum += c[i];
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (ln >= o) incl += v;
    }
    int excl = incl - lsum;
    const uint32_t hit = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (ln == src) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (excl + c[i] >= remaining) {
          digit = 255 - 8 * ln - i;
          above = excl;
          break;
        }
        excl += c[i];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    remaining -= above;
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
    __syncwarp();
  }
  *kth = prefix;
  *need = remaining;
}

template <int R>
__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int RT = R >= 16 ? R / 16 : 1;  // rows per thread in the logit tile
  constexpr int KS = 65;                    // padded stride of the transposed K chunk
  const int D = a.d, QS = D + 1;
  const int Tq = a.Tq, Tk = a.Tkv;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int row0 = blockIdx.x * R;
  float* qs = reinterpret_cast<float*>(sm);           // [R][D+1]
  float* kt = qs + R * QS;                            // [D][KS]
  uint32_t* hist = reinterpret_cast<uint32_t*>(kt + D * KS);  // [8][256]
  uint32_t* keys = hist + 8 * 256;                    // [R][Tk]
  const float* Qc = a.Qc + (int64_t)bh * Tq * D;
  const float* Kc = a.Kc + (int64_t)bh * Tk * D;
  for (int e = tid; e < R * D; e += 256) {
    const int r = e / D, c = e % D;
    qs[r * QS + c] = (row0 + r < Tq) ? Qc[(int64_t)(row0 + r) * D + c] : 0.f;
  }
  // K_c chunk of 64 key blocks: thread e loads the 4 columns 4q..4q+3 of row
  // jj = e % 64 (q = e / 64), so a warp's transposed stores hit 32 banks.
  constexpr int NV = 64 * 32 / 256;  // float4 loads per thread for d = 128 (8); d = 64 uses 4
  const int nv = (64 * (D / 4)) / 256;
  float4 pre[NV];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      if (v < nv) {
        const int e = tid + 256 * v, jj = e & 63, q = e >> 6;
        pre[v] = (j0 + jj < Tk) ? __ldg(reinterpret_cast<const float4*>(Kc + (int64_t)(j0 + jj) * D) + q)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  load_chunk(0);
  const float scale = rsqrtf((float)D);
  const int ty = tid >> 4, tx = tid & 15;
  const bool rows_ok = (R >= 16) || ty < R;
  for (int j0 = 0; j0 < Tk; j0 += 64) {
    __syncthreads();
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      if (v < nv) {
        const int e = tid + 256 * v, jj = e & 63, q = e >> 6;
        kt[(4 * q + 0) * KS + jj] = pre[v].x;
        kt[(4 * q + 1) * KS + jj] = pre[v].y;
        kt[(4 * q + 2) * KS + jj] = pre[v].z;
        kt[(4 * q + 3) * KS + jj] = pre[v].w;
      }
    }
    __syncthreads();
    if (j0 + 64 < Tk) load_chunk(j0 + 64);  // next chunk in flight during the math
    if (rows_ok) {
      float acc[RT][4];
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
#pragma unroll 4
      for (int k = 0; k < D; ++k) {
        float qv[RT];
#pragma unroll
        for (int i = 0; i < RT; ++i) qv[i] = qs[(ty + 16 * i) * QS + k];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float kv = kt[k * KS + tx + 16 * c];
#pragma unroll
          for (int i = 0; i < RT; ++i) acc[i][c] = fmaf(qv[i], kv, acc[i][c]);
        }
      }
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = j0 + tx + 16 * c;
          if (j < Tk) keys[(ty + 16 * i) * Tk + j] = order_key(acc[i][c] * scale);
        }
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << ln) - 1u;
  for (int rr = w; rr < R; rr += 8) {
    const int i = row0 + rr;
    if (i >= Tq) break;
    const uint32_t* rk = keys + rr * Tk;
    // critical: top n_h; kept (critical or marginal): top T_kv - n_l
    uint32_t kh, kk;
    int need_h, need_k;
    kth_largest(rk, Tk, a.nh, hist + w * 256, &kh, &need_h);
    kth_largest(rk, Tk, Tk - a.nl, hist + w * 256, &kk, &need_k);
    int8_t* mrow = a.mc + ((int64_t)bh * Tq + i) * Tk;
    int32_t* lrow = a.lut + ((int64_t)bh * Tq + i) * a.nh;
    int eq_h = 0, eq_k = 0, ncrit = 0;
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
  const size_t smem = (size_t)(D * 68 + D * (D + 1)) * sizeof(float);
  cudaError_t e;
  if (D == 128) {
    e = cudaFuncSetAttribute(router_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    router_kernel<128><<<dim3((Tq + 63) / 64, BH), 256, smem, s>>>(Qc, nullptr, Wq, Qr, Tq);
    router_kernel<128><<<dim3((Tk + 63) / 64, BH), 256, smem, s>>>(Kc, smooth ? kmean : nullptr, Wk, Kr, Tk);
  } else {
    e = cudaFuncSetAttribute(router_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    router_kernel<64><<<dim3((Tq + 63) / 64, BH), 256, smem, s>>>(Qc, nullptr, Wq, Qr, Tq);
    router_kernel<64><<<dim3((Tk + 63) / 64, BH), 256, smem, s>>>(Kc, smooth ? kmean : nullptr, Wk, Kr, Tk);
  }
  return cudaGetLastError();
}

// Rows of logits per CTA: at most what ~150 KB of keys allow (32, 16 or 8),
// fewer when that leaves too few CTAs to fill the GPU twice over.
static int select_rows(int Tq, int Tk, int BH) {
  int R = Tk <= 1200 ? 32 : (Tk <= 2400 ? 16 : 8);
  while (R > 8 && (int64_t)((Tq + R - 1) / R) * BH < 2 * 148) R /= 2;
  return R;
}

static size_t select_smem_bytes_r(int R, int D, int Tk) {
  return (size_t)(R * (D + 1) + D * 65) * sizeof(float) + 8 * 256 * 4 + (size_t)R * Tk * 4;
}

size_t select_smem_bytes(int D, int Tk) { return select_smem_bytes_r(Tk <= 1200 ? 32 : (Tk <= 2400 ? 16 : 8), D, Tk); }

template <int R>
static cudaError_t launch_select_t(const SelectArgs& a, int BH, cudaStream_t s) {
  const size_t smem = select_smem_bytes_r(R, a.d, a.Tkv);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<R><<<dim3((a.Tq + R - 1) / R, BH), 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, int BH, cudaStream_t s) {
  const int R = select_rows(a.Tq, a.Tkv, BH);
  if (R == 32) return launch_select_t<32>(a, BH, s);
  if (R == 16) return launch_select_t<16>(a, BH, s);
  return launch_select_t<8>(a, BH, s);
}

}  // namespace sla
