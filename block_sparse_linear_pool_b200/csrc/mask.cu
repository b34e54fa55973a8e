// Compressed mask prediction ("SLA: Beyond Sparsity in Diffusion Transformers
// via Fine-Tunable Sparse-Linear Attention", §2 Q2 steps 1-2 and Fig. 4 left;
// "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §4):
//   pool_kernel     mean of Q and K over 64-token blocks (real tokens only)
//   kmean_kernel    token mean of K per head (smooth-K, SLA §7 item 3)
//   router_kernel   x <- (x - mean) W^T for the SLA2 router projections (fp32)
//   logits_kernel   keys = order-preserving 32-bit form of Q_c K_c^T / sqrt(d),
//                   fp32 tiled GEMM
//   select_kernel   exact row-wise top-n_h / bottom-n_l selection by radix
//                   search over the keys, one warp per row
#include "kernels.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// pool: one warp per 64-token block.  Each lane loads 16 bytes (8 columns) of a
// row per instruction, so one instruction covers 32 * 16 / (2 D) rows (2 for
// d = 128, 4 for d = 64); 8 loads per lane are in flight (few enough registers
// for six CTAs per SM).  Lanes holding the
// same columns of different rows are summed with shuffles at the end.
// grid (ceil(T/8), B*H, 2): z = 0 pools Q into Qc, z = 1 pools K into Kc.
// Rows start on 16-byte boundaries (base and token stride are checked by the
// entry points).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256, 6) pool_kernel(PoolArgs a) {
  constexpr int LPR = D / 8;        // lanes per row: 16 (d=128) or 8 (d=64)
  constexpr int RPI = 32 / LPR;     // rows per instruction: 2 or 4
  const int w = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int blk = blockIdx.x * 8 + w;
  const int bh = blockIdx.y;
  const int T = a.T;
  if (blk >= T) return;
  const int b = bh / a.H, h = bh % a.H;
  const __nv_bfloat16* src = blockIdx.z == 0 ? a.Q : a.K;
  const int64_t* st = blockIdx.z == 0 ? a.sq : a.sk;
  float* dst = blockIdx.z == 0 ? a.Qc : a.Kc;
  const int t0 = blk * a.bs;
  const int cnt = min(a.bs, a.N - t0);
  const int roff = ln / LPR, col = (ln % LPR) * 8;
  const __nv_bfloat16* base = src + (int64_t)b * st[0] + (int64_t)h * st[1] + (int64_t)t0 * st[2] + col;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  auto add = [&](const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __low2float(p[e]);
      acc[2 * e + 1] += __high2float(p[e]);
    }
  };
  if (cnt == 64) {
    // whole block: 64 / RPI rows per lane, loaded in groups of 16 before use
    constexpr int PER = 64 / RPI;
    constexpr int G = PER < 8 ? PER : 8;
#pragma unroll
    for (int g0 = 0; g0 < PER; g0 += G) {
      uint4 v[G];
#pragma unroll
      for (int i = 0; i < G; ++i)
        v[i] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(roff + RPI * (g0 + i)) * st[2]));
#pragma unroll
      for (int i = 0; i < G; ++i) add(v[i]);
    }
  } else {
    for (int t = roff; t < cnt; t += RPI)
      add(__ldg(reinterpret_cast<const uint4*>(base + (int64_t)t * st[2])));
  }
#pragma unroll
  for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], m);
  if (roff == 0) {
    const float inv = 1.f / (float)cnt;
    float4* out = reinterpret_cast<float4*>(dst + ((int64_t)bh * T + blk) * D + col);
    out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
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
// logits: keys[bh][i][j] = order_key(Q_c[i] . K_c[j] / sqrt(d)) in fp32 (fp32
// keeps the logits exact to ~1e-6, far inside the 1e-4 grading gap; bf16
// tensor cores would not).  64 x 128 tile per CTA (so that a 512 x 512 head
// gives 32 CTAs and the grid fills every SM more than twice), d consumed in
// chunks of 32 through two shared-memory stages (the next chunk's loads are in
// flight while the current one is multiplied).
// grid (ceil(T_kv/128), ceil(T_q/64), B*H).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

namespace {
constexpr int LM = 64, LN = 128, LK = 32;  // tile rows (queries), columns (keys), k chunk
constexpr int LAS = LM + 4, LBS = LN + 4;  // padded strides
constexpr int LOGITS_SMEM = 2 * LK * (LAS + LBS) * (int)sizeof(float);  // two stages: 51 KB
}

__global__ void __launch_bounds__(256) logits_kernel(LogitArgs a) {
  extern __shared__ __align__(16) float lsm[];
  float* As = lsm;                  // [2][LK][LAS]
  float* Bs = lsm + 2 * LK * LAS;   // [2][LK][LBS]
  const int D = a.d, Tq = a.Tq, Tk = a.Tkv, bh = blockIdx.z;
  const int m0 = blockIdx.y * LM, n0 = blockIdx.x * LN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const float* A = a.Qc + (int64_t)bh * Tq * D;
  const float* B = a.Kc + (int64_t)bh * Tk * D;
  // staging: element e of a tile is row e % rows, column quad e / rows (a warp
  // covers 32 rows of one quad, so the transposed stores hit distinct banks)
  constexpr int NA = LM * LK / 4 / 256, NB = LN * LK / 4 / 256;  // float4 per thread: 2, 4
  float4 pa[NA], pb[NB];
  auto load = [&](int k0) {
#pragma unroll
    for (int v = 0; v < NA; ++v) {
      const int e = tid + 256 * v, r = e % LM, q = e / LM;
      pa[v] = (m0 + r < Tq) ? __ldg(reinterpret_cast<const float4*>(A + (int64_t)(m0 + r) * D + k0) + q)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int v = 0; v < NB; ++v) {
      const int e = tid + 256 * v, r = e % LN, q = e / LN;
      pb[v] = (n0 + r < Tk) ? __ldg(reinterpret_cast<const float4*>(B + (int64_t)(n0 + r) * D + k0) + q)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int st) {
    float* as = As + st * LK * LAS;
    float* bs = Bs + st * LK * LBS;
#pragma unroll
    for (int v = 0; v < NA; ++v) {
      const int e = tid + 256 * v, r = e % LM, q = e / LM;
      as[(4 * q + 0) * LAS + r] = pa[v].x;
      as[(4 * q + 1) * LAS + r] = pa[v].y;
      as[(4 * q + 2) * LAS + r] = pa[v].z;
      as[(4 * q + 3) * LAS + r] = pa[v].w;
    }
#pragma unroll
    for (int v = 0; v < NB; ++v) {
      const int e = tid + 256 * v, r = e % LN, q = e / LN;
      bs[(4 * q + 0) * LBS + r] = pb[v].x;
      bs[(4 * q + 1) * LBS + r] = pb[v].y;
      bs[(4 * q + 2) * LBS + r] = pb[v].z;
      bs[(4 * q + 3) * LBS + r] = pb[v].w;
    }
  };
  // thread (ty, tx) owns rows 4ty..4ty+3 and columns {4tx..4tx+3, 64+4tx..64+4tx+3},
  // accumulated in column pairs with the paired fp32 FMA (each half rounded as fmaf)
  uint64_t acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;
  load(0);
  store(0);
  __syncthreads();
  const int nk = D / LK;
  for (int kc = 0; kc < nk; ++kc) {
    const int st = kc & 1;
    if (kc + 1 < nk) load((kc + 1) * LK);
    const float* as = As + st * LK * LAS;
    const float* bs = Bs + st * LK * LBS;
#pragma unroll
    for (int k = 0; k < LK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(as + k * LAS + 4 * ty);
      const float4 b0 = *reinterpret_cast<const float4*>(bs + k * LBS + 4 * tx);
      const float4 b1 = *reinterpret_cast<const float4*>(bs + k * LBS + 64 + 4 * tx);
      const float av[4] = {a0.x, a0.y, a0.z, a0.w};
      const uint64_t bp[4] = {f2_pack(b0.x, b0.y), f2_pack(b0.z, b0.w), f2_pack(b1.x, b1.y), f2_pack(b1.z, b1.w)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t ap = f2_pack(av[i], av[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = f2_fma(ap, bp[j], acc[i][j]);
      }
    }
    if (kc + 1 < nk) store(st ^ 1);
    __syncthreads();
  }
  const float scale = rsqrtf((float)D);
  uint32_t* keys = a.keys + (int64_t)bh * Tq * Tk;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + 4 * ty + i;
    if (r >= Tq) continue;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      float v[2];
      f2_unpack(acc[i][jj], v[0], v[1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * jj + h;
        const int c = n0 + (j < 4 ? 4 * tx + j : 64 + 4 * tx + (j - 4));
        if (c < Tk) keys[(int64_t)r * Tk + c] = order_key(v[h] * scale);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// select: one warp per (head, query block) row.  The row's keys are copied to
// shared memory.  The n_h-th largest and the (T_kv - n_l)-th largest keys are
// found exactly in two steps:
//   1. a 256-bin histogram of the logit VALUES over [row min, row max]
//      (bin = floor((x - min) * 256 / (max - min)), clamped: non-decreasing in
//      x, so every key of a higher bin is larger than every key of a lower
//      one); a descending scan gives, for each rank, its bin and how many keys
//      lie in the bins above;
//   2. the keys of that bin (a few for any spread-out row) are ranked among
//      themselves: directly when they fit one warp, else by an exact
//      most-significant-bit-first radix search with counts by warp reduction.
// Ties rank the lower block index first.  One row per warp, up to 8 warps per
// CTA (fewer when T_kv is large, to keep two CTAs' keys in shared memory).
// ---------------------------------------------------------------------------
struct RadixState {
  uint32_t prefix, mask;
  int remaining;
};

__device__ __forceinline__ void radix_step(RadixState& st, int bit, int cnt) {
  const uint32_t cand = st.prefix | (1u << bit);
  if (cnt >= st.remaining) {
    st.prefix = cand;
  } else {
    st.remaining -= cnt;
  }
  st.mask |= 1u << bit;
}

// Bits `hi`..0 of one search over n keys.
__device__ void radix_rounds1(const uint32_t* keys, int n, int hi, RadixState& A) {
  const int ln = threadIdx.x & 31;
  for (int bit = hi; bit >= 0; --bit) {
    const uint32_t ma = A.mask | (1u << bit), ca = A.prefix | (1u << bit);
    int na = 0;
    for (int j = ln; j < n; j += 32) na += ((keys[j] & ma) == ca);
    radix_step(A, bit, __reduce_add_sync(0xffffffffu, na));
  }
}

// The inverse of order_key (keys of -0 and +0 are one key, read back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ int value_bin(uint32_t k, float xmin, float inv) {
  // NaN (0 * inf when the range underflows) goes to bin 0 through fmaxf
  return (int)fminf(fmaxf((key_value(k) - xmin) * inv, 0.f), 255.f);
}

// The `rank`-th largest of the m keys in `list` (1 <= rank <= m): returns the
// key and, in *take, how many of the keys equal to it rank within `rank`; *eq
// is how many keys of the list equal it (0 when not counted).
__device__ uint32_t rank_in_list(const uint32_t* list, int m, int rank, int* take, int* eq) {
  const int ln = threadIdx.x & 31;
  if (m <= 32) {
    const uint32_t mine = ln < m ? list[ln] : 0u;
    int gt = 0, ge = 0;
    for (int j = 0; j < m; ++j) {
      const uint32_t o = __shfl_sync(0xffffffffu, mine, j);
      gt += o > mine;
      ge += o >= mine;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, ln < m && gt < rank && rank <= ge);
    const int src = __ffs(hit) - 1;  // every hit lane holds the same key
    const uint32_t key = __shfl_sync(0xffffffffu, mine, src);
    const int g = __shfl_sync(0xffffffffu, gt, src);
    *take = rank - g;
    *eq = __shfl_sync(0xffffffffu, ge, src) - g;
    return key;
  }
  *eq = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j = ln; j < m; j += 32) {
    kmin = min(kmin, list[j]);
    kmax = max(kmax, list[j]);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // every key of the list shares the bits above the highest bit where min and max differ
  const uint32_t diff = kmin ^ kmax;
  const int top_bit = diff ? 31 - __clz(diff) : -1;
  const uint32_t shared_mask = top_bit >= 31 ? 0u : (top_bit < 0 ? 0xffffffffu : ~((2u << top_bit) - 1u));
  RadixState st = {kmin & shared_mask, shared_mask, rank};
  if (top_bit >= 0) radix_rounds1(list, m, top_bit, st);
  *take = st.remaining;
  return st.prefix;
}

// Keys of `src` (n) in value bin b0 to d0 and in bin b1 (!= b0) to d1, in order.
__device__ void compact_bins(const uint32_t* src, int n, int b0, int b1, float xmin, float inv, uint32_t* d0,
                             uint32_t* d1) {
  const int ln = threadIdx.x & 31;
  const uint32_t lt = (1u << ln) - 1u;
  int m0 = 0, m1 = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + ln;
    const uint32_t key = j < n ? src[j] : 0u;
    const int b = j < n ? value_bin(key, xmin, inv) : -1;
    const uint32_t bal0 = __ballot_sync(0xffffffffu, b == b0);
    const uint32_t bal1 = __ballot_sync(0xffffffffu, b == b1);
    if (b == b0) d0[m0 + __popc(bal0 & lt)] = key;
    if (b == b1) d1[m1 + __popc(bal1 & lt)] = key;
    m0 += __popc(bal0);
    m1 += __popc(bal1);
  }
  __syncwarp();
}

// The bin of the `rank`-th largest key from the descending per-lane bin counts
// c (lane l holds bins 255 - 8l - i, i = 0..7), and the number of keys above it.
__device__ __forceinline__ int scan_bin(const int (&c)[8], int incl, int sum, int rank, int* above) {
  const int ln = threadIdx.x & 31;
  const uint32_t reach = __ballot_sync(0xffffffffu, incl >= rank);
  const int L = __ffs(reach) - 1;
  int bin = 0, ab = 0;
  if (ln == L) {
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (run + c[i] >= rank) {
        bin = 255 - 8 * ln - i;
        ab = run;
        break;
      }
      run += c[i];
    }
  }
  *above = __shfl_sync(0xffffffffu, ab, L);
  return __shfl_sync(0xffffffffu, bin, L);
}

__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  // per warp: keys [T_kv], candidates [T_kv], histogram [256]
  extern __shared__ __align__(16) uint32_t skeys[];
  const int Tq = a.Tq, Tk = a.Tkv;
  const int w = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + w;  // bh * Tq + i
  if (row >= (int64_t)a.BH * Tq) return;
  uint32_t* rk = skeys + (int64_t)w * (2 * Tk + 256);
  uint32_t* cand = rk + Tk;
  int* hist = reinterpret_cast<int*>(cand + Tk);
  const uint32_t* g = a.keys + row * Tk;
#pragma unroll
  for (int i = 0; i < 8; ++i) hist[8 * ln + i] = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j = ln; j < Tk; j += 32) {
    const uint32_t v = g[j];
    rk[j] = v;
    kmin = min(kmin, v);
    kmax = max(kmax, v);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncwarp();
  // A: the n_h-th largest (critical); B: the (T_kv - n_l)-th largest (kept)
  const int rank_h = a.nh, rank_k = Tk - a.nl;
  uint32_t kh = kmax, kk = kmax;
  int need_h = rank_h, need_k = rank_k;
  int eq_h_all = 0, eq_k_all = 0;  // keys equal to each threshold (0: not counted)
  if (kmin != kmax) {
    const float xmin = key_value(kmin);
    const float inv = 256.f / (key_value(kmax) - xmin);
    for (int j = ln; j < Tk; j += 32) atomicAdd(&hist[value_bin(rk[j], xmin, inv)], 1);
    __syncwarp();
    int c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = hist[255 - 8 * ln - i];
      sum += c[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (ln >= o) incl += y;
    }
    int above_h, above_k;
    const int bin_h = scan_bin(c, incl, sum, rank_h, &above_h);
    const int bin_k = scan_bin(c, incl, sum, rank_k, &above_k);
    // the bins' sizes are in the histogram: both candidate lists fit `cand`
    const int m_h = hist[bin_h], m_k = hist[bin_k];
    uint32_t* cand_k = bin_k == bin_h ? cand : cand + m_h;
    compact_bins(rk, Tk, bin_h, bin_k == bin_h ? -2 : bin_k, xmin, inv, cand, cand_k);
    kh = rank_in_list(cand, m_h, rank_h - above_h, &need_h, &eq_h_all);
    kk = rank_in_list(cand_k, m_k, rank_k - above_k, &need_k, &eq_k_all);
  }
  int8_t* mrow = a.mc + row * Tk;
  int32_t* lrow = a.lut + row * a.nh;
  const uint32_t lt = (1u << ln) - 1u;
  int eq_h = 0, eq_k = 0, ncrit = 0;
  if (eq_h_all == 1 && eq_k_all == 1) {
    // no ties at either threshold: every key at or above a threshold is in
    for (int j0 = 0; j0 < Tk; j0 += 32) {
      const int j = j0 + ln;
      const bool valid = j < Tk;
      const uint32_t key = valid ? rk[j] : 0u;
      const bool crit = valid && key >= kh;
      const uint32_t bc = __ballot_sync(0xffffffffu, crit);
      if (valid) mrow[j] = crit ? (int8_t)1 : (key >= kk ? (int8_t)0 : (int8_t)-1);
      if (crit) lrow[ncrit + __popc(bc & lt)] = j;
      ncrit += __popc(bc);
    }
    return;
  }
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

// Rows (warps) per select CTA: at most 8, and at most ~112 KB of keys.
int select_rows_per_cta(int Tk) {
  int r = 8;
  while (r > 1 && (size_t)r * (2 * Tk + 256) * sizeof(uint32_t) > (size_t)112 * 1024) r >>= 1;
  return r;
}

size_t select_smem_bytes(int Tk) {
  return (size_t)select_rows_per_cta(Tk) * (2 * Tk + 256) * sizeof(uint32_t);
}

cudaError_t launch_logits(const LogitArgs& la, int BH, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LOGITS_SMEM);
  if (e != cudaSuccess) return e;
  logits_kernel<<<dim3((la.Tkv + LN - 1) / LN, (la.Tq + LM - 1) / LM, BH), 256, LOGITS_SMEM, s>>>(la);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, int BH, cudaStream_t s) {
  LogitArgs la;
  la.Qc = a.Qc;
  la.Kc = a.Kc;
  la.keys = a.keys;
  la.d = a.d;
  la.Tq = a.Tq;
  la.Tkv = a.Tkv;
  cudaError_t e = launch_logits(la, BH, s);
  if (e != cudaSuccess) return e;
  const size_t smem = select_smem_bytes(a.Tkv);
  e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  SelectArgs b = a;
  b.BH = BH;
  const int64_t rows = (int64_t)BH * a.Tq;
  const int r = select_rows_per_cta(a.Tkv);
  select_kernel<<<(unsigned)((rows + r - 1) / r), 32 * r, smem, s>>>(b);
  return cudaGetLastError();
}

}  // namespace sla
