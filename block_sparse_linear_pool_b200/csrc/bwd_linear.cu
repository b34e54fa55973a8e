// Backward of the linear branch and of the combine ("SLA2: Sparse-Linear
// Attention with Learnable Routing and QAT", App. A; "SLA: Beyond Sparsity in
// Diffusion Transformers via Fine-Tunable Sparse-Linear Attention", §4 check 6:
// the linear branch's gradients go through per-query-block dH_i, dZ_i that
// are accumulated into the marginal key blocks, mirroring the forward).
//
// Notation.  W~ = Proj's W (SLA) or the identity (SLA2); c_s, c_l = 1, 1 (SLA)
// or alpha, 1 - alpha (SLA2).  The forward's statistics carry W~ already:
// H'_i = H_i W~^T, so o'_r = phi(q_r) H'_i / den_r = o_l W~^T with
// den_r = phi(q_r) . Z_i + eps.  Every linear-branch gradient can be written
// with the primed quantities, so the unprojected H_i is never formed:
//   gp_r    = c_l dO_r / den_r                  (= g_r W~^T with g_r = do_l / den_r)
//   gden_r  = -c_l (dO_r . o'_r) / den_r
//   dphi(q_r) = H'_i gp_r + gden_r Z_i
//   dH'_i   = sum_r phi(q_r)^T gp_r,  dZ_i = sum_r gden_r phi(q_r)
//   dh'_j   = sum of dH'_i over the query blocks that have j marginal (a GEMM)
//   u_t     = dh'_j^T phi(k_t)          dv_t (linear) = W~^T u_t
//   dphi(k_t) = dh'_j (W~ v_t) + dz_j   dW = sum_t u_t v_t^T
// and for the sparse branch's backward (o^s from the forward, fp32):
// D_r = c_s dO_r . o^s_r; SLA2's d alpha = sum_r (o^s_r - o'_r) . dO_r.
//
//   bwd_rows_kernel   one query block per CTA: D, dq (linear part, fp32),
//                     [dH'_i | dZ_i] (bf16, the layout of the forward's
//                     [H_i^T | Z_i]), d alpha and d bias partial sums
//   bwd_keys_kernel   persistent over key blocks: dk, dv (linear parts, fp32)
//                     and dW (held per CTA in registers, added once at the end)
//
// Both are plain fp32 FMA kernels: 64 x d x d products staged in shared memory.
#include "kernels.cuh"

namespace sla {
namespace {

constexpr float LOG2E = 1.4426950408889634f;

// phi over d for one 64-row tile held one row per warp pass: x (fp32, row of D)
// -> f written to dst.  Lane l owns columns l, l+32, ...
template <int D>
__device__ __forceinline__ void feature_row(const float* x, float* f, int phi) {
  constexpr int PL = D / 32;
  const int ln = threadIdx.x & 31;
  float v[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) v[u] = x[ln + 32 * u];
  if (phi == 1) {
#pragma unroll
    for (int u = 0; u < PL; ++u) f[ln + 32 * u] = v[u] > 0.f ? v[u] + 1.f : exp2f(v[u] * LOG2E);
    return;
  }
  float m = v[0];
#pragma unroll
  for (int u = 1; u < PL; ++u) m = fmaxf(m, v[u]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    v[u] = exp2f((v[u] - m) * LOG2E);
    s += v[u];
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.f / s;
#pragma unroll
  for (int u = 0; u < PL; ++u) f[ln + 32 * u] = v[u] * inv;
}

// acc[i][j] += sum_k A(r_i, k) B(k, c_j) over k < K for the thread's 4 x CT tile
// of a 64 x D product: rows r_i = 4 ty + i, columns c_j = tx + 16 j
// (ty = tid / 16, tx = tid % 16, 256 threads; interleaved columns keep the
// sixteen threads of a half-warp on distinct shared-memory banks).
template <int CT, class FA, class FB>
__device__ __forceinline__ void tile_mma(float (&acc)[4][CT], int K, FA A, FB Bm) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float a[4], bv[CT];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = A(4 * ty + i, k);
#pragma unroll
    for (int j = 0; j < CT; ++j) bv[j] = Bm(k, tx + 16 * j);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
  }
}

template <int CT>
__device__ __forceinline__ void zero(float (&acc)[4][CT]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
}

__device__ __forceinline__ float bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

}  // namespace

// ---------------------------------------------------------------------------
// Query side.  grid (T_q, B*H), 256 threads.
// Shared: F = phi(Q) [64][D], G = gp [64][D], Hs = H'_i as bf16 [o][a] with
// rows padded to D + 2 (bank-conflict-free column reads), Z [D], den / gden [64].
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_rows_kernel(BwdRowsArgs a) {
  constexpr int CT = D / 16;
  constexpr int LD = D + 2;
  extern __shared__ float sm[];
  float* F = sm;                 // [64][D]
  float* G = F + 64 * D;         // [64][D]
  __nv_bfloat16* Hs = reinterpret_cast<__nv_bfloat16*>(G + 64 * D);  // [D][LD]: Hs[o][a] = H'_i[a][o]
  float* Z = reinterpret_cast<float*>(Hs + D * LD);                   // [D]
  float* den = Z + D;            // [64]
  float* gden = den + 64;        // [64]
  float* red = gden + 64;        // [8 warps][D + 1]
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int n0 = 64 * i;
  const int rows = min(64, a.N - n0);
  const float cs = a.combine == 1 ? a.alpha[bh] : 1.f;
  const float cl = a.combine == 1 ? 1.f - a.alpha[bh] : 1.f;

  // [H'_i^T | Z_i]: row element o*D + a holds H'_i[a][o], element D*D + a holds Z_i[a]
  const __nv_bfloat16* hz = a.hagg + ((int64_t)bh * a.Tq + i) * a.NN;
  for (int e = tid; e < D * D; e += 256) Hs[(e / D) * LD + (e % D)] = hz[e];
  for (int e = tid; e < D; e += 256) Z[e] = bf(hz + D * D + e);
  // phi(q_r), one row per warp pass (rows past N are zero)
  for (int r = w; r < 64; r += 8) {
    float* fr = F + r * D;
    if (r < rows) {
      const __nv_bfloat16* q = a.Q + (int64_t)b * a.sq[0] + (int64_t)h * a.sq[1] + (int64_t)(n0 + r) * a.sq[2];
      float* x = G + r * D;  // scratch for the raw row
      for (int c = ln; c < D; c += 32) x[c] = bf(q + c);
      __syncwarp();
      feature_row<D>(x, fr, a.phi);
    } else {
      for (int c = ln; c < D; c += 32) fr[c] = 0.f;
    }
  }
  __syncthreads();
  // NUM = phi(Q) H'_i  (64 x D):  NUM[r][o] = sum_a F[r][a] Hs[o][a]
  float acc[4][CT];
  zero(acc);
  tile_mma<CT>(acc, D, [&](int r, int k) { return F[r * D + k]; },
               [&](int k, int c) { return bf(Hs + c * LD + k); });
  // den_r = phi(q_r) . Z_i + eps
  for (int r = w; r < 64; r += 8) {
    float s = 0.f;
    for (int c = ln; c < D; c += 32) s += F[r * D + c] * Z[c];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (ln == 0) den[r] = s + a.eps;
  }
  __syncthreads();
  // o'_r = NUM / den into G (scratch), then per row: o^s, D, gp, gden, d alpha, d bias
  {
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int r = 4 * ty + ii;
      const float inv = 1.f / den[r];
#pragma unroll
      for (int j = 0; j < CT; ++j) G[r * D + tx + 16 * j] = acc[ii][j] * inv;
    }
  }
  __syncthreads();
  float dalpha_part = 0.f;
  float* dbias = red;  // [8][D] partial column sums of dO (SLA)
  for (int c = ln; c < D; c += 32) dbias[w * (D + 1) + c] = 0.f;
  for (int r = w; r < 64; r += 8) {
    float* g = G + r * D;
    if (r >= rows) {
      for (int c = ln; c < D; c += 32) g[c] = 0.f;
      if (ln == 0) {
        gden[r] = 0.f;
        a.ld2[(int64_t)bh * a.Tq * 64 + n0 + r] = make_float2(-INFINITY, 0.f);  // P = 0 there
      }
      continue;
    }
    const int64_t n = n0 + r;
    const float* orow = a.os + ((int64_t)bh * a.N + n) * D;
    const __nv_bfloat16* drow = a.dO + (int64_t)b * a.so[0] + (int64_t)h * a.so[1] + n * a.so[2];
    float dd = 0.f, dol = 0.f, da = 0.f;
    for (int c = ln; c < D; c += 32) {
      const float ol = g[c];                       // o'_r
      const float dov = bf(drow + c);
      const float os = orow[c];                    // o^s_r
      dd += cs * dov * os;
      dol += dov * ol;
      da += (os - ol) * dov;
      g[c] = cl * dov / den[r];                    // gp_r
      if (a.combine == 0) dbias[w * (D + 1) + c] += dov;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      dd += __shfl_xor_sync(0xffffffffu, dd, o);
      dol += __shfl_xor_sync(0xffffffffu, dol, o);
      da += __shfl_xor_sync(0xffffffffu, da, o);
    }
    if (ln == 0) {
      a.ld2[(int64_t)bh * a.Tq * 64 + n] = make_float2(-a.lse[(int64_t)bh * a.N + n] * LOG2E, -dd);
      gden[r] = -cl * dol / den[r];
    }
    dalpha_part += da;
  }
  __syncthreads();
  if (a.combine == 1 && a.dalpha && ln == 0) atomicAdd(a.dalpha + bh, dalpha_part);
  if (a.combine == 0 && a.dproj_b) {
    for (int c = tid; c < D; c += 256) {
      float s = 0.f;
      for (int ww = 0; ww < 8; ++ww) s += dbias[ww * (D + 1) + c];
      atomicAdd(a.dproj_b + c, s);
    }
  }
  // dphi(q) = gp H'^T + gden Z:  dphi[r][a] = sum_o G[r][o] Hs[o][a] + gden[r] Z[a]
  zero(acc);
  tile_mma<CT>(acc, D, [&](int r, int k) { return G[r * D + k]; },
               [&](int k, int c) { return bf(Hs + k * LD + c); });
  // dH'_i = F^T G (D x D, k = rows) and dZ_i = gden^T F, written before G is reused
  {
    // dH'[a][o] = sum_r F[r][a] G[r][o]; tile rows = a (64 at a time), columns = o
    __nv_bfloat16* out = a.dhz + ((int64_t)bh * a.Tq + i) * a.NN;
    for (int a0 = 0; a0 < D; a0 += 64) {
      float acc2[4][CT];
      zero(acc2);
      tile_mma<CT>(acc2, 64, [&](int r, int k) { return F[k * D + a0 + r]; },
                   [&](int k, int c) { return G[k * D + c]; });
      const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int j = 0; j < CT; ++j) {
          const int aa = a0 + 4 * ty + ii, o = tx + 16 * j;
          out[(int64_t)o * D + aa] = __float2bfloat16(acc2[ii][j]);  // [o][a] like the forward
        }
    }
    for (int c = tid; c < D; c += 256) {
      float s = 0.f;
      for (int r = 0; r < 64; ++r) s += gden[r] * F[r * D + c];
      out[D * D + c] = __float2bfloat16(s);
    }
  }
  __syncthreads();
  {
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int r = 4 * ty + ii;
#pragma unroll
      for (int j = 0; j < CT; ++j) {
        const int c = tx + 16 * j;
        G[r * D + c] = acc[ii][j] + gden[r] * Z[c];  // dphi(q_r)
      }
    }
  }
  __syncthreads();
  // dq (linear part) = phi backward, fp32 into the scratch
  for (int r = w; r < rows; r += 8) {
    const int64_t n = n0 + r;
    const __nv_bfloat16* q = a.Q + (int64_t)b * a.sq[0] + (int64_t)h * a.sq[1] + n * a.sq[2];
    float x[D / 32], dx[D / 32];
    float* outq = a.dq_lin + ((int64_t)bh * a.N + n) * D;
#pragma unroll
    for (int u = 0; u < D / 32; ++u) x[u] = bf(q + ln + 32 * u);
    const float* f = F + r * D;
    const float* df = G + r * D;
    if (a.phi == 1) {
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const int c = ln + 32 * u;
        dx[u] = df[c] * (x[u] > 0.f ? 1.f : f[c]);
      }
    } else {
      float dot = 0.f;
#pragma unroll
      for (int u = 0; u < D / 32; ++u) dot += f[ln + 32 * u] * df[ln + 32 * u];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const int c = ln + 32 * u;
        dx[u] = f[c] * (df[c] - dot);
      }
    }
#pragma unroll
    for (int u = 0; u < D / 32; ++u) outq[ln + 32 * u] = dx[u];
  }
}

// ---------------------------------------------------------------------------
// Key side.  Persistent: grid min(#blocks, SMs), 256 threads; CTA c takes key
// blocks c, c + G, ...  Shared: Ws = W~ [o][c] fp32 with rows padded to D + 1,
// Gs = dh'_j as bf16 [o][a] with rows padded to D + 2, X1 = phi(K_j),
// X2 = V_j then dphi(k), X3 = u then w = W~ v.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_keys_kernel(BwdKeysArgs a) {
  constexpr int CT = D / 16;
  constexpr int LD = D + 1, LG = D + 2;
  extern __shared__ float sm[];
  float* Ws = sm;                // [D][LD]
  __nv_bfloat16* Gs = reinterpret_cast<__nv_bfloat16*>(Ws + D * LD);  // [D][LG]: Gs[o][a] = dh'_j[a][o]
  float* X1 = reinterpret_cast<float*>(Gs + D * LG);                  // [64][D]
  float* X2 = X1 + 64 * D;       // [64][D]
  float* X3 = X2 + 64 * D;       // [64][D]
  float* Zs = X3 + 64 * D;       // [D]: dz_j
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int tx = tid & 15, ty = tid >> 4;
  const bool proj = a.proj_w != nullptr;
  for (int e = tid; e < D * D; e += 256)
    Ws[(e / D) * LD + (e % D)] = proj ? a.proj_w[e] : ((e / D) == (e % D) ? 1.f : 0.f);
  // dW partial: this thread owns dW[o][c] for o = 64 hh + 4 ty + i (hh < D / 64),
  // c = tx + 16 j
  constexpr int NHALF = D / 64;
  float dw[NHALF][4][CT];
#pragma unroll
  for (int hh = 0; hh < NHALF; ++hh) zero(dw[hh]);
  const int nblocks = a.BH * a.Tkv;
  for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const int bh = blk / a.Tkv, j = blk % a.Tkv;
    const int b = bh / a.H, h = bh % a.H;
    const int n0 = 64 * j, rows = min(64, a.N - n0);
    __syncthreads();  // the previous block's buffers are free
    const __nv_bfloat16* g = a.dhz + ((int64_t)bh * a.Tkv + j) * a.NN;
    for (int e = tid; e < D * D; e += 256) Gs[(e / D) * LG + (e % D)] = g[e];
    for (int e = tid; e < D; e += 256) Zs[e] = bf(g + D * D + e);
    for (int r = w; r < 64; r += 8) {
      if (r < rows) {
        const int64_t n = n0 + r;
        const __nv_bfloat16* kr = a.K + (int64_t)b * a.sk[0] + (int64_t)h * a.sk[1] + n * a.sk[2];
        const __nv_bfloat16* vr = a.V + (int64_t)b * a.sv[0] + (int64_t)h * a.sv[1] + n * a.sv[2];
        for (int c = ln; c < D; c += 32) {
          X3[r * D + c] = bf(kr + c);
          X2[r * D + c] = bf(vr + c);
        }
        __syncwarp();
        feature_row<D>(X3 + r * D, X1 + r * D, a.phi);
      } else {
        for (int c = ln; c < D; c += 32) X1[r * D + c] = X2[r * D + c] = 0.f;
      }
    }
    __syncthreads();
    // u = phi(K) dh'_j:  u[t][o] = sum_a X1[t][a] Gs[o][a]
    float acc[4][CT];
    zero(acc);
    tile_mma<CT>(acc, D, [&](int r, int k) { return X1[r * D + k]; },
                 [&](int k, int c) { return bf(Gs + c * LG + k); });
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < CT; ++jj) X3[(4 * ty + ii) * D + tx + 16 * jj] = acc[ii][jj];
    __syncthreads();
    // dW += u^T V:  dW[o][c] = sum_t u[t][o] V[t][c]
    if (proj) {
#pragma unroll
      for (int hh = 0; hh < NHALF; ++hh)
        tile_mma<CT>(dw[hh], 64, [&](int r, int k) { return X3[k * D + 64 * hh + r]; },
                     [&](int k, int c) { return X2[k * D + c]; });
    }
    // dv (linear) = u W~:  dv[t][c] = sum_o u[t][o] Ws[o][c]
    zero(acc);
    tile_mma<CT>(acc, D, [&](int r, int k) { return X3[r * D + k]; },
                 [&](int k, int c) { return Ws[k * LD + c]; });
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int r = 4 * ty + ii;
      if (r < rows) {
        float* out = a.dv_lin + ((int64_t)bh * a.N + n0 + r) * D;
#pragma unroll
        for (int jj = 0; jj < CT; ++jj) out[tx + 16 * jj] = acc[ii][jj];
      }
    }
    // w = V W~^T:  w[t][o] = sum_c V[t][c] Ws[o][c]  (into X3: u is no longer needed)
    __syncthreads();
    zero(acc);
    tile_mma<CT>(acc, D, [&](int r, int k) { return X2[r * D + k]; },
                 [&](int k, int c) { return Ws[c * LD + k]; });
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < CT; ++jj) X3[(4 * ty + ii) * D + tx + 16 * jj] = acc[ii][jj];
    __syncthreads();
    // dphi(k) = w dh'_j^T + dz_j:  dphi[t][a] = sum_o X3[t][o] Gs[o][a] + Zs[a]
    zero(acc);
    tile_mma<CT>(acc, D, [&](int r, int k) { return X3[r * D + k]; },
                 [&](int k, int c) { return bf(Gs + k * LG + c); });
    __syncthreads();
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < CT; ++jj) {
        const int c = tx + 16 * jj;
        X2[(4 * ty + ii) * D + c] = acc[ii][jj] + Zs[c];  // V is no longer needed
      }
    __syncthreads();
    // dk (linear) = phi backward
    for (int r = w; r < rows; r += 8) {
      const int64_t n = n0 + r;
      const __nv_bfloat16* kr = a.K + (int64_t)b * a.sk[0] + (int64_t)h * a.sk[1] + n * a.sk[2];
      const float* f = X1 + r * D;
      const float* df = X2 + r * D;
      float* out = a.dk_lin + ((int64_t)bh * a.N + n) * D;
      if (a.phi == 1) {
        for (int c = ln; c < D; c += 32) out[c] = df[c] * (bf(kr + c) > 0.f ? 1.f : f[c]);
      } else {
        float dot = 0.f;
        for (int c = ln; c < D; c += 32) dot += f[c] * df[c];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        for (int c = ln; c < D; c += 32) out[c] = f[c] * (df[c] - dot);
      }
    }
  }
  if (proj && a.dproj_w) {
#pragma unroll
    for (int hh = 0; hh < NHALF; ++hh)
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < CT; ++jj)
          atomicAdd(a.dproj_w + (64 * hh + 4 * ty + ii) * D + tx + 16 * jj, dw[hh][ii][jj]);
  }
}

size_t bwd_rows_smem(int D) {
  return (size_t)(2 * 64 * D + D + 128 + 8 * (D + 1)) * 4 + (size_t)D * (D + 2) * 2;
}
size_t bwd_keys_smem(int D) {
  return (size_t)(D * (D + 1) + 3 * 64 * D + D) * 4 + (size_t)D * (D + 2) * 2;
}

cudaError_t launch_bwd_rows(const BwdRowsArgs& a, int D, int BH, cudaStream_t s) {
  const size_t smem = bwd_rows_smem(D);
  dim3 grid(a.Tq, BH);
  if (D == 128) {
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_rows_kernel<128><<<grid, 256, smem, s>>>(a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_rows_kernel<64><<<grid, 256, smem, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_keys(const BwdKeysArgs& a, int D, cudaStream_t s) {
  const size_t smem = bwd_keys_smem(D);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nblocks = a.BH * a.Tkv;
  const int grid = nblocks < sms ? nblocks : sms;
  if (D == 128) {
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_keys_kernel<128><<<grid, 256, smem, s>>>(a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_keys_kernel<64><<<grid, 256, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sla
