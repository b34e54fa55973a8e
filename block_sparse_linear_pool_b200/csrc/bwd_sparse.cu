// Backward of the sparse branch ("SLA: Beyond Sparsity in Diffusion
// Transformers via Fine-Tunable Sparse-Linear Attention", §4 check 6: the
// sparse path's gradients follow the FlashAttention backward; §7: one kernel
// for dQ and one for dK / dV).  Only critical (query block, key block) pairs
// are visited, as in the forward.
//
// With P = exp(s - lse) the forward's probabilities over a row's critical
// tokens (lse from the forward), dP = dO^s V^T, D_r = dO^s_r . o^s_r and
// dS = P (dP - D):   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),  dV = P^T dO^s,
// where dO^s = c_s dO (c_s = 1 for SLA, alpha for SLA2; applied to dP and to
// the finished dV).  The linear branch's parts (fp32, from the linear
// backward) are added in the epilogues.
//
//   rlut_*              reverse lists: for every key block, the query blocks
//                       that have it critical (ascending), from M_c
//   bwd_dq_kernel       CTA = two query blocks (M = 128; the forward's pairing
//                       by critical-list overlap) over the union of their
//                       critical lists: S = Q K^T and dP = dO V^T into
//                       TMEM (two buffers), dS by the row threads, dQ += dS K
//                       (dS read from TMEM)
//   bwd_dkdv_kernel     CTA = two key blocks (M = 128 key rows, paired by
//                       reverse-list overlap) over the union of their reverse
//                       lists: S^T = K Q^T and
//                       dP^T = V dO^T into TMEM (two buffers), P^T and dS^T by
//                       the key-row threads, dV += P^T dO and dK += dS^T Q
// Both: warp 0 TMA producer, warp 1 MMA issuer, warps 2-9 two threads per TMEM
// lane (each takes half of the 64 columns of a score tile).
#include "kernels.cuh"

namespace sla {

namespace {

__device__ __forceinline__ float ex2b(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
}  // namespace

// ---------------------------------------------------------------------------
// Reverse lists.  rcnt[bh][j] = #query blocks with M_c = 1 at column j; rptr =
// exclusive prefix sums (rptr[bh][T_kv] = T_q * n_h); rows = the query block
// indices, ascending per column.
// ---------------------------------------------------------------------------
__global__ void rlut_count_kernel(const int8_t* __restrict__ mc, int32_t* __restrict__ rcnt, int Tq,
                                  int Tkv) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
  if (j >= Tkv) return;
  const int8_t* col = mc + (int64_t)bh * Tq * Tkv + j;
  int c = 0;
  for (int i = 0; i < Tq; ++i) c += col[(int64_t)i * Tkv] == 1;
  rcnt[(int64_t)bh * Tkv + j] = c;
}

__global__ void __launch_bounds__(1024) rlut_scan_kernel(const int32_t* __restrict__ rcnt,
                                                         int32_t* __restrict__ rptr, int Tkv) {
  __shared__ int32_t part[1024];
  const int bh = blockIdx.x, t = threadIdx.x;
  const int per = (Tkv + 1023) / 1024;
  const int j0 = t * per;
  int s = 0;
  for (int j = j0; j < min(j0 + per, Tkv); ++j) s += rcnt[(int64_t)bh * Tkv + j];
  part[t] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan of the per-thread sums
    const int v = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = t > 0 ? part[t - 1] : 0;
  int32_t* out = rptr + (int64_t)bh * (Tkv + 1);
  for (int j = j0; j < min(j0 + per, Tkv); ++j) {
    out[j] = run;
    run += rcnt[(int64_t)bh * Tkv + j];
  }
  if (t == 1023) out[Tkv] = part[1023];
}

__global__ void rlut_fill_kernel(const int8_t* __restrict__ mc, const int32_t* __restrict__ rptr,
                                 int32_t* __restrict__ rows, int Tq, int Tkv, int nh) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
  if (j >= Tkv) return;
  const int8_t* col = mc + (int64_t)bh * Tq * Tkv + j;
  int32_t* out = rows + (int64_t)bh * Tq * nh + rptr[(int64_t)bh * (Tkv + 1) + j];
  int k = 0;
  for (int i = 0; i < Tq; ++i)
    if (col[(int64_t)i * Tkv] == 1) out[k++] = i;
}

cudaError_t launch_rlut(const int8_t* mc, int32_t* rcnt, int32_t* rptr, int32_t* rows, int BH,
                        int Tq, int Tkv, int nh, cudaStream_t s) {
  dim3 grid((Tkv + 127) / 128, BH);
  rlut_count_kernel<<<grid, 128, 0, s>>>(mc, rcnt, Tq, Tkv);
  rlut_scan_kernel<<<BH, 1024, 0, s>>>(rcnt, rptr, Tkv);
  rlut_fill_kernel<<<grid, 128, 0, s>>>(mc, rptr, rows, Tq, Tkv, nh);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// dQ.  TMEM (512 columns, one CTA per SM): two score buffers x = 0, 1 with S at
// [128x, 128x + 64) (dS over its first 32 columns) and dP at [128x + 64,
// 128x + 128); dQ at [256, 256 + d); the CTA's Q and dO rows (bf16 pairs) at
// [384, 384 + d/2) and [448, 448 + d/2).  S, dP of entry k+1 are computed while
// the row threads turn entry k into dS.  S = Q K^T and dP = dO V^T take Q and
// dO from TMEM and only the 64-key tile from shared memory; an M = 128, N = 64
// MMA costs about the same either way (some 65 cycles per K = 16 step), and
// this form measured about 1% faster than both operands in shared memory.  Shared: Q and dO tiles (128 rows), a
// 4-slot K ring (K_k serves S_k and, later, dQ += dS_k K_k) and a 3-slot V ring.
// ---------------------------------------------------------------------------
template <int D>
struct DqSmem {
  static constexpr int CH = D / 64;
  static constexpr int T128 = 128 * D * 2;
  static constexpr int T64 = 64 * D * 2;
  static constexpr int NK = 4, NV = 3;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + T128;
  static constexpr int OFF_K = OFF_DO + T128;
  static constexpr int OFF_V = OFF_K + NK * T64;
  static constexpr int OFF_BAR = OFF_V + NV * T64;
  static constexpr int OFF_U = OFF_BAR + 256;
  // at least 120 KB: one CTA per SM (it holds all 512 TMEM columns)
  static size_t bytes(int Tkv) {
    const size_t b = (size_t)OFF_U + 5 * (size_t)((Tkv + 15) & ~15) + 1024;
    return b < 120 * 1024 ? 120 * 1024 : b;
  }
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapdO,
                  const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                  BwdSparseArgs a) {
  using L = DqSmem<D>;
  constexpr int NK = L::NK, NV = L::NV;
  constexpr uint32_t COL_DQ = 256, COL_Q = 384, COL_DO = 448;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sdO = sm + L::OFF_DO;
  uint8_t* sK = sm + L::OFF_K;
  uint8_t* sV = sm + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* in_full = bars + 0;          // Q and dO
  uint64_t* k_full = bars + 1;           // [NK]
  uint64_t* k_empty = k_full + NK;       // [NK]
  uint64_t* v_full = k_empty + NK;       // [NV]
  uint64_t* v_empty = v_full + NV;       // [NV]
  uint64_t* sp_full = v_empty + NV;      // [2] S and dP of buffer x
  uint64_t* ds_ready = sp_full + 2;      // [2] dS written by all row threads
  uint64_t* dq_done = ds_ready + 2;      // the last dQ MMA completed
  uint64_t* qt_ready = dq_done + 1;      // Q and dO copied into TMEM by the row threads
  uint32_t* tslot = reinterpret_cast<uint32_t*>(qt_ready + 1);
  int* s_count = reinterpret_cast<int*>(tslot + 1);
  const int Tkvr = (a.Tkv + 15) & ~15;
  uint8_t* fa = sm + L::OFF_U;
  uint8_t* fb = fa + Tkvr;
  uint8_t* uflag = fb + Tkvr;
  uint16_t* uidx = reinterpret_cast<uint16_t*>(uflag + Tkvr);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  // the CTA's two query blocks (rows 0-63: ia, rows 64-127: ib); ib < 0: none
  const int2 pair = a.pairs[(int64_t)bh * ((a.Tq + 1) / 2) + p];
  const int ia = pair.x, ib = pair.y;
  const bool has_b = ib >= 0;
  const int ibl = has_b ? ib : ia;  // block loaded into the second half

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(in_full, 1);
    for (int x = 0; x < NK; ++x) {
      mbar_init(&k_full[x], 1);
      mbar_init(&k_empty[x], 1);
    }
    for (int x = 0; x < NV; ++x) {
      mbar_init(&v_full[x], 1);
      mbar_init(&v_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sp_full[x], 1);
      mbar_init(&ds_ready[x], 8);
    }
    mbar_init(dq_done, 1);
    mbar_init(qt_ready, 8);
    fence_barrier_init();
  }
  for (int j = tid; j < 2 * Tkvr; j += blockDim.x) fa[j] = 0;
  __syncthreads();
  if (tid == 0) {  // the Q and dO tiles do not depend on the union: load them while it is built
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapdO);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    mbar_arrive_expect_tx(in_full, 2 * L::T128);
#pragma unroll
    for (int c = 0; c < L::CH; ++c) {
      tma_load_4d(sQ + c * 16384, &mapQ, in_full, c * 64, 64 * ia, h, b);
      tma_load_4d(sQ + c * 16384 + 8192, &mapQ, in_full, c * 64, 64 * ibl, h, b);
      tma_load_4d(sdO + c * 16384, &mapdO, in_full, c * 64, 64 * ia, h, b);
      tma_load_4d(sdO + c * 16384 + 8192, &mapdO, in_full, c * 64, 64 * ibl, h, b);
    }
  }
  {
    const int32_t* la = a.lut + ((int64_t)bh * a.Tq + ia) * a.nh;
    const int32_t* lb = a.lut + ((int64_t)bh * a.Tq + ibl) * a.nh;
    const int tot = has_b ? 2 * a.nh : a.nh;
    for (int e = tid; e < tot; e += blockDim.x) {
      const bool second = e >= a.nh;
      const int j = second ? lb[e - a.nh] : la[e];
      if (j < 0 || j >= a.Tkv) {
        atomicCAS(a.err, 0, DEV_BAD_INDEX);
        continue;
      }
      (second ? fb : fa)[j] = 1;
    }
  }
  __syncthreads();
  if (w == 0) {
    int base = 0;
    const uint32_t lt = (1u << ln) - 1u;
    for (int j0 = 0; j0 < a.Tkv; j0 += 32) {
      const int j = j0 + ln;
      const uint32_t f = (j < a.Tkv) ? (uint32_t)(fa[j] | (fb[j] << 1)) : 0u;
      const uint32_t bal = __ballot_sync(0xffffffffu, f != 0);
      if (f) {
        const int pos = base + __popc(bal & lt);
        uidx[pos] = (uint16_t)j;
        uflag[pos] = (uint8_t)f;
      }
      base += __popc(bal);
    }
    if (ln == 0) *s_count = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int U = *s_count;
  const uint32_t tbase = *tslot;

  if (w == 0) {
    if (ln == 0) {
      bool ok = true;
      for (int k = 0; k < U && ok; ++k) {
        const int j = uidx[k], sk = k % NK, sv = k % NV;
        if (k >= NK && !mbar_wait(&k_empty[sk], ((k / NK) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[sk], L::T64);
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_load_4d(sK + sk * L::T64 + c * 8192, &mapK, &k_full[sk], c * 64, 64 * j, h, b);
        if (k >= NV && !mbar_wait(&v_empty[sv], ((k / NV) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[sv], L::T64);
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_load_4d(sV + sv * L::T64 + c * 8192, &mapV, &v_full[sv], c * 64, 64 * j, h, b);
      }
    }
  } else if (w == 1) {
    if (ln == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_q = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(qt_ready, 0, a.err, DEV_TIMEOUT_SYNC);
      // dQ += dS_k K_k: dS (bf16 pairs) from TMEM buffer k & 1, K as the MN-major B operand
      auto issue_dq = [&](int k) -> bool {
        const int x = k & 1, sk = k % NK;
        if (!mbar_wait(&ds_ready[x], (k >> 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        tc_fence_after();
        // descriptors advanced by constants: a byte offset o adds o >> 4
        const uint64_t dk = sdesc_sw128(smem_u32(sK), 8192, 1024) + (uint64_t)(sk * L::T64 >> 4);
        // keys 16 kk .. 16 kk + 15: packed at columns 32 (kk / 2) + 8 (kk % 2)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tbase + COL_DQ, tbase + 128 * x + 32 * (kk / 2) + 8 * (kk % 2), dk + kk * (2048 >> 4), id_q,
                  (k > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&k_empty[sk]);
        return true;
      };
      for (int k = 0; k < U && ok; ++k) {
        const int x = k & 1, sk = k % NK, sv = k % NV;
        if (!mbar_wait(&k_full[sk], (k / NK) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
        if (!mbar_wait(&v_full[sv], (k / NV) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
        tc_fence_after();
        // S and dP into buffer x; its previous contents (entry k - 2) were consumed
        // by the dQ MMA issued earlier by this thread (in-order execution).  Q and dO
        // from TMEM: d = 16 kk .. 16 kk + 15 at columns 8 kk .. 8 kk + 7.
        const uint64_t dkt = sdesc_sw128(smem_u32(sK), 16, 1024) + (uint64_t)(sk * L::T64 >> 4);
        const uint64_t dvt = sdesc_sw128(smem_u32(sV), 16, 1024) + (uint64_t)(sv * L::T64 >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = ((kk / 4) * 8192 + (kk % 4) * 32) >> 4;
          umma_ts(tbase + 128 * x, tbase + COL_Q + 8 * kk, dkt + offk, id_s, kk > 0 ? 1u : 0u);
          umma_ts(tbase + 128 * x + 64, tbase + COL_DO + 8 * kk, dvt + offk, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sp_full[x]);
        umma_commit(&v_empty[sv]);
        if (k >= 1 && !issue_dq(k - 1)) { ok = false; break; }
      }
      if (ok && U >= 1) ok = issue_dq(U - 1);
      if (ok) umma_commit(dq_done);
    }
  } else {
    // ---------------- two threads per query row (warps w and w + 4 share TMEM
    // lanes); each turns 32 of the 64 key columns into dS
    const int q4 = w & 3;
    const int hs = (w - 2) >> 2;
    const int r = 32 * q4 + ln;
    const int half = r >> 6;
    const uint32_t bit = 1u << half;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    const int n = 64 * (half == 0 ? ia : ibl) + (r & 63);
    const bool valid = (n < a.N) && (half == 0 || has_b);
    // (-lse log2 e, -D) of this row; P = 0 on rows that do not exist
    const float2 ld = valid ? a.ld2[(int64_t)bh * a.Tq * 64 + n] : make_float2(-INFINITY, 0.f);
    const float cs = a.combine == 1 ? a.alpha[bh] : 1.f;
    const float sl2 = a.scale_log2;
    // paired constants: P = 2^(s sl2 - lse2), dS = P (cs dP - D)
    const uint64_t sc2 = f2_pack(sl2, sl2), nl2 = f2_pack(ld.x, ld.x), cs2 = f2_pack(cs, cs),
                   nd2 = f2_pack(ld.y, ld.y);
    // this thread's half of the row's fp32 linear part, added in the epilogue
    const float* lin = a.q_lin + ((int64_t)bh * a.N + n) * D + (D / 2) * hs;
    // this thread's half of the row's Q and dO (d = (D/2) hs ..) from the swizzled
    // tiles into TMEM as bf16 pairs, the A operands of the S and dP MMAs
    bool ok = __all_sync(0xffffffffu, mbar_wait(in_full, 0, a.err, DEV_TIMEOUT_TMA));
    if (ok) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint8_t* src = which == 0 ? sQ : sdO;
        uint32_t qv[D / 4];
#pragma unroll
        for (int u = 0; u < D / 16; ++u) {  // 16-byte units: 8 bf16 = 4 columns each
          const int d0 = (D / 2) * hs + 8 * u;
          const uint4 t = *reinterpret_cast<const uint4*>(src + (d0 / 64) * 16384 + sw128_offset(r, (d0 % 64) * 2));
          qv[4 * u] = t.x;
          qv[4 * u + 1] = t.y;
          qv[4 * u + 2] = t.z;
          qv[4 * u + 3] = t.w;
        }
        const uint32_t col = (which == 0 ? COL_Q : COL_DO) + (D / 4) * hs;
        if constexpr (D == 128) {
          tmem_st32(tl + col, qv);
        } else {
          tmem_st16(tl + col, qv);
        }
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (ok && ln == 0) mbar_arrive(qt_ready);
    for (int k = 0; k < U && ok; ++k) {
      const int x = k & 1;
      if (valid && k == (U > 3 ? U - 3 : 0)) {  // into L2 a few entries ahead of the epilogue
#pragma unroll
        for (int c = 0; c < D / 2; c += 32) prefetch_l2(lin + c);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sp_full[x], (k >> 1) & 1, a.err, DEV_TIMEOUT_MMA))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool crit = (uflag[k] & bit) != 0;
      const uint32_t ts = tl + 128 * x;
      uint32_t pk[16];
      if (crit) {
        uint32_t s0[32], d0[32];
        tmem_ld32(ts + 32 * hs, s0);
        tmem_ld32(ts + 64 + 32 * hs, d0);
        tmem_ld_wait();
        const int nvalid = a.N - 64 * (int)uidx[k] - 32 * hs;  // warp-uniform
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2, nl2), x0, x1);
          float p0 = ex2b(x0), p1 = ex2b(x1);
          if (nvalid < 32) {  // columns past N (the last key block) have P = 0
            p0 = 2 * c < nvalid ? p0 : 0.f;
            p1 = 2 * c + 1 < nvalid ? p1 : 0.f;
          }
          const uint64_t g = f2_fma(f2_pack(__uint_as_float(d0[2 * c]), __uint_as_float(d0[2 * c + 1])), cs2, nd2);
          float d0s, d1s;
          f2_unpack(f2_mul(f2_pack(p0, p1), g), d0s, d1s);
          pk[c] = pack_bf16x2(d0s, d1s);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = 0u;
      }
      // dS for this thread's 32 keys (16 bf16 pairs) over the start of its own S
      // columns: the other thread of the row never reads them
      tmem_st16(ts + 32 * hs, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (ln == 0) mbar_arrive(&ds_ready[x]);  // one arrival per warp
    }
    if (ok && U >= 1) ok = __all_sync(0xffffffffu, mbar_wait(dq_done, 0, a.err, DEV_TIMEOUT_MMA));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* orow = a.out0 + (int64_t)b * a.s0[0] + (int64_t)h * a.s0[1] + (int64_t)n * a.s0[2] +
                            (D / 2) * hs;
      // all of this thread's linear part in flight before the first TMEM read
      float4 lv[D / 8];
#pragma unroll
      for (int q = 0; q < D / 8; ++q)
        lv[q] = valid ? __ldg(reinterpret_cast<const float4*>(lin) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {  // this thread's half of the row
        uint32_t v[32];
        if (U >= 1) {
          tmem_ld32(tl + COL_DQ + (D / 2) * hs + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const float4 l0 = lv[c0 / 4 + 2 * q8], l1 = lv[c0 / 4 + 2 * q8 + 1];
            const float* vf = reinterpret_cast<const float*>(v + 8 * q8);
            *reinterpret_cast<uint4*>(orow + c0 + 8 * q8) =
                make_uint4(pack_bf16x2(vf[0] * a.scale + l0.x, vf[1] * a.scale + l0.y),
                           pack_bf16x2(vf[2] * a.scale + l0.z, vf[3] * a.scale + l0.w),
                           pack_bf16x2(vf[4] * a.scale + l1.x, vf[5] * a.scale + l1.y),
                           pack_bf16x2(vf[6] * a.scale + l1.z, vf[7] * a.scale + l1.w));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// dK, dV.  TMEM (512 columns, one CTA per SM): two score buffers x = 0, 1 with
// S^T at [128x, 128x + 64) (P^T over its first 32 columns) and dP^T at
// [128x + 64, 128x + 128) (dS^T over its first 32), dV [256, 256 + d),
// dK [384, 384 + d).  S^T, dP^T of entry e+1 are computed while the key-row
// threads work on entry e.  Shared: K pair and V pair (128 rows), a 4-slot
// ring of (Q_i, dO_i, the 64 (lse log2 e, D) pairs of block i).  A slot is
// freed only when the dV / dK MMAs of its entry complete, one entry after its
// S^T; with two slots the load of entry e + 2 could start only then, and the
// tensor pipe waited out a whole load every entry.
// ---------------------------------------------------------------------------
template <int D>
struct DkvSmem {
  static constexpr int CH = D / 64;
  static constexpr int T128 = 128 * D * 2;
  static constexpr int T64 = 64 * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + T128;
  static constexpr int NQ = 4;                      // ring slots
  static constexpr int OFF_Q = OFF_V + T128;        // [NQ] slots
  static constexpr int OFF_DO = OFF_Q + NQ * T64;   // [NQ]
  static constexpr int OFF_LD = OFF_DO + NQ * T64;  // [NQ][64] float2
  static constexpr int OFF_BAR = OFF_LD + NQ * 64 * 8;
  static constexpr int OFF_U = OFF_BAR + 256;
  // at least 120 KB so that a second CTA (which would wait for the 512 TMEM
  // columns) is never placed on the same SM
  static size_t bytes(int Tq) {
    const size_t b = (size_t)OFF_U + 5 * (size_t)((Tq + 15) & ~15) + 1024;
    return b < 120 * 1024 ? 120 * 1024 : b;
  }
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mapK2, const __grid_constant__ CUtensorMap mapV2,
                    const __grid_constant__ CUtensorMap mapQ1, const __grid_constant__ CUtensorMap mapdO1,
                    BwdSparseArgs a) {
  using L = DkvSmem<D>;
  constexpr uint32_t COL_DV = 256, COL_DK = 384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sK = sm + L::OFF_K;
  uint8_t* sV = sm + L::OFF_V;
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sdO = sm + L::OFF_DO;
  float2* sLD = reinterpret_cast<float2*>(sm + L::OFF_LD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  constexpr int NQ = L::NQ;
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;             // [NQ] ring slots
  uint64_t* q_empty = q_full + NQ;         // [NQ]
  uint64_t* sp_full = q_empty + NQ;        // [2] score buffers
  uint64_t* ds_ready = sp_full + 2;        // [2]
  uint64_t* kv_done = ds_ready + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(kv_done + 1);
  int* s_count = reinterpret_cast<int*>(tslot + 1);
  const int Tqr = (a.Tq + 15) & ~15;
  uint8_t* fa = sm + L::OFF_U;
  uint8_t* fb = fa + Tqr;
  uint8_t* uflag = fb + Tqr;
  uint16_t* uidx = reinterpret_cast<uint16_t*>(uflag + Tqr);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  // the CTA's two key blocks (rows 0-63: ja, rows 64-127: jb); jb < 0: none
  const int2 pair = a.pairs[(int64_t)bh * ((a.Tkv + 1) / 2) + p];
  const int ja = pair.x, jb = pair.y;
  const bool has_b = jb >= 0;
  const int jbl = has_b ? jb : ja;  // block loaded into the second half

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int x = 0; x < NQ; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sp_full[x], 1);
      mbar_init(&ds_ready[x], 8);
    }
    mbar_init(kv_done, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < 2 * Tqr; i += blockDim.x) fa[i] = 0;
  __syncthreads();
  if (tid == 0) {  // the K and V pair does not depend on the union: load it while it is built
    tma_prefetch_desc(&mapK2);
    tma_prefetch_desc(&mapV2);
    tma_prefetch_desc(&mapQ1);
    tma_prefetch_desc(&mapdO1);
    mbar_arrive_expect_tx(kv_full, 2 * L::T128);
#pragma unroll
    for (int c = 0; c < L::CH; ++c) {
      tma_load_4d(sK + c * 16384, &mapK2, kv_full, c * 64, 64 * ja, h, b);
      tma_load_4d(sK + c * 16384 + 8192, &mapK2, kv_full, c * 64, 64 * jbl, h, b);
      tma_load_4d(sV + c * 16384, &mapV2, kv_full, c * 64, 64 * ja, h, b);
      tma_load_4d(sV + c * 16384 + 8192, &mapV2, kv_full, c * 64, 64 * jbl, h, b);
    }
  }
  {
    const int32_t* rp = a.rptr + (int64_t)bh * (a.Tkv + 1);
    const int32_t* rl = a.rows + (int64_t)bh * a.Tq * a.nh;
    for (int t = 0; t < (has_b ? 2 : 1); ++t) {
      const int j = t == 0 ? ja : jb;
      const int e0 = rp[j], e1 = rp[j + 1];
      for (int e = e0 + tid; e < e1; e += blockDim.x) {
        const int i = rl[e];
        if (i < 0 || i >= a.Tq) {
          atomicCAS(a.err, 0, DEV_BAD_INDEX);
          continue;
        }
        (t == 0 ? fa : fb)[i] = 1;
      }
    }
  }
  __syncthreads();
  if (w == 0) {
    int base = 0;
    const uint32_t lt = (1u << ln) - 1u;
    for (int i0 = 0; i0 < a.Tq; i0 += 32) {
      const int i = i0 + ln;
      const uint32_t f = (i < a.Tq) ? (uint32_t)(fa[i] | (fb[i] << 1)) : 0u;
      const uint32_t bal = __ballot_sync(0xffffffffu, f != 0);
      if (f) {
        const int pos = base + __popc(bal & lt);
        uidx[pos] = (uint16_t)i;
        uflag[pos] = (uint8_t)f;
      }
      base += __popc(bal);
    }
    if (ln == 0) *s_count = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int U = *s_count;
  const uint32_t tbase = *tslot;

  if (w == 0) {
    if (ln == 0) {
      bool ok = true;
      for (int e = 0; e < U && ok; ++e) {
        const int i = uidx[e], sq = e % NQ;
        if (e >= NQ && !mbar_wait(&q_empty[sq], ((e / NQ) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[sq], 2 * L::T64 + 64 * 8);
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_load_4d(sQ + sq * L::T64 + c * 8192, &mapQ1, &q_full[sq], c * 64, 64 * i, h, b);
          tma_load_4d(sdO + sq * L::T64 + c * 8192, &mapdO1, &q_full[sq], c * 64, 64 * i, h, b);
        }
        bulk_load(sLD + sq * 64, a.ld2 + (int64_t)bh * a.Tq * 64 + 64 * i, 64 * 8, &q_full[sq]);
      }
    }
  } else if (w == 1) {
    if (ln == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_o = idesc_bf16(128, D, false, true);
      const uint32_t k0 = smem_u32(sK), v0 = smem_u32(sV);
      bool ok = mbar_wait(kv_full, 0, a.err, DEV_TIMEOUT_TMA);
      // dV += P^T dO_e and dK += dS^T Q_e (P^T, dS^T bf16 pairs from TMEM buffer e & 1)
      auto issue_grads = [&](int e) -> bool {
        const int x = e & 1, sq = e % NQ;
        if (!mbar_wait(&ds_ready[x], (e >> 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        tc_fence_after();
        // descriptors advanced by constants: a byte offset o adds o >> 4
        const uint64_t dqt = sdesc_sw128(smem_u32(sQ), 8192, 1024) + (uint64_t)(sq * L::T64 >> 4);
        const uint64_t dot = sdesc_sw128(smem_u32(sdO), 8192, 1024) + (uint64_t)(sq * L::T64 >> 4);
        // query rows 16 kk .. 16 kk + 15: packed at columns 32 (kk / 2) + 8 (kk % 2)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ca = 32 * (kk / 2) + 8 * (kk % 2);
          umma_ts(tbase + COL_DV, tbase + 128 * x + ca, dot + kk * (2048 >> 4), id_o, (e > 0 || kk > 0) ? 1u : 0u);
          umma_ts(tbase + COL_DK, tbase + 128 * x + 64 + ca, dqt + kk * (2048 >> 4), id_o,
                  (e > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&q_empty[sq]);
        return true;
      };
      for (int e = 0; e < U && ok; ++e) {
        const int x = e & 1, sq = e % NQ;
        if (!mbar_wait(&q_full[sq], (e / NQ) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
        tc_fence_after();
        // S^T = K Q_e^T and dP^T = V dO_e^T (M = 128 key rows, N = 64 query rows) into
        // buffer x; its previous contents (entry e - 2) were consumed by MMAs issued
        // earlier by this thread, which execute in order
        const uint64_t dk0 = sdesc_sw128(k0, 16, 1024), dv0 = sdesc_sw128(v0, 16, 1024);
        const uint64_t dqt = sdesc_sw128(smem_u32(sQ), 16, 1024) + (uint64_t)(sq * L::T64 >> 4);
        const uint64_t dot = sdesc_sw128(smem_u32(sdO), 16, 1024) + (uint64_t)(sq * L::T64 >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off2 = ((kk / 4) * 16384 + (kk % 4) * 32) >> 4, off1 = ((kk / 4) * 8192 + (kk % 4) * 32) >> 4;
          umma_ss(tbase + 128 * x, dk0 + off2, dqt + off1, id_s, kk > 0 ? 1u : 0u);
          umma_ss(tbase + 128 * x + 64, dv0 + off2, dot + off1, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sp_full[x]);
        if (e >= 1 && !issue_grads(e - 1)) { ok = false; break; }
      }
      if (ok && U >= 1) ok = issue_grads(U - 1);
      if (ok) umma_commit(kv_done);
    }
  } else {
    // ---------------- two threads per key row (warps w and w + 4 share TMEM
    // lanes); each handles 32 of the 64 query columns
    const int q4 = w & 3;
    const int hs = (w - 2) >> 2;
    const int t = 32 * q4 + ln;
    const int half = t >> 6;
    const uint32_t bit = 1u << half;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    const int n = 64 * (half == 0 ? ja : jbl) + (t & 63);
    const bool valid = (n < a.N) && (half == 0 || has_b);
    const float cs = a.combine == 1 ? a.alpha[bh] : 1.f;
    const float sl2 = a.scale_log2;
    // this thread's halves of the key row's fp32 linear parts (dK, dV), added in the epilogue
    const float* lin_k = a.q_lin + ((int64_t)bh * a.N + n) * D + (D / 2) * hs;
    const float* lin_v = a.v_lin + ((int64_t)bh * a.N + n) * D + (D / 2) * hs;
    bool ok = true;
    for (int e = 0; e < U; ++e) {
      const int x = e & 1;
      if (valid && e == (U > 3 ? U - 3 : 0)) {  // into L2 a few entries ahead of the epilogue
#pragma unroll
        for (int c = 0; c < D / 2; c += 32) {
          prefetch_l2(lin_k + c);
          prefetch_l2(lin_v + c);
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sp_full[x], (e >> 1) & 1, a.err, DEV_TIMEOUT_MMA))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool crit = (uflag[e] & bit) != 0;
      const uint32_t ts = tl + 128 * x;
      uint32_t pp[16], pd[16];
      if (crit) {
        uint32_t s0[32], d0[32];
        tmem_ld32(ts + 32 * hs, s0);
        tmem_ld32(ts + 64 + 32 * hs, d0);
        tmem_ld_wait();
        // (-lse log2 e, -D) of this thread's 32 query rows
        const float4* ldv = reinterpret_cast<const float4*>(sLD + (e % NQ) * 64 + 32 * hs);
        const uint64_t sc2 = f2_pack(sl2, sl2), cs2 = f2_pack(cs, cs);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float4 l4 = ldv[c];  // rows 2c and 2c + 1
          float p0, p1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2,
                           f2_pack(l4.x, l4.z)), p0, p1);
          p0 = ex2b(p0);
          p1 = ex2b(p1);
          const uint64_t g = f2_fma(f2_pack(__uint_as_float(d0[2 * c]), __uint_as_float(d0[2 * c + 1])), cs2,
                                    f2_pack(l4.y, l4.w));
          float d0s, d1s;
          f2_unpack(f2_mul(f2_pack(p0, p1), g), d0s, d1s);
          pp[c] = pack_bf16x2(p0, p1);
          pd[c] = pack_bf16x2(d0s, d1s);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) pp[c] = pd[c] = 0u;
      }
      // P^T and dS^T for this thread's 32 query rows over the start of its own
      // S^T and dP^T columns (the other thread of the row never reads them)
      tmem_st16(ts + 32 * hs, pp);
      tmem_st16(ts + 64 + 32 * hs, pd);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (ln == 0) mbar_arrive(&ds_ready[x]);  // one arrival per warp
    }
    if (ok && U >= 1) ok = __all_sync(0xffffffffu, mbar_wait(kv_done, 0, a.err, DEV_TIMEOUT_MMA));
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* base = which == 0 ? a.out0 : a.out1;
        const int64_t* st = which == 0 ? a.s0 : a.s1;
        const float* lin = which == 0 ? lin_k : lin_v;
        const float f = which == 0 ? a.scale : cs;  // dK = acc / sqrt(d); dV = c_s acc
        __nv_bfloat16* orow = base + (int64_t)b * st[0] + (int64_t)h * st[1] + (int64_t)n * st[2] + (D / 2) * hs;
        const uint32_t col = (which == 0 ? COL_DK : COL_DV) + (D / 2) * hs;
        // all of this half row's linear part in flight before the first TMEM read
        float4 lv[D / 8];
#pragma unroll
        for (int q = 0; q < D / 8; ++q)
          lv[q] = valid ? __ldg(reinterpret_cast<const float4*>(lin) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t v[32];
          if (U >= 1) {
            tmem_ld32(tl + col + c0, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = 0u;
          }
          if (valid) {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              const float4 l0 = lv[c0 / 4 + 2 * q8], l1 = lv[c0 / 4 + 2 * q8 + 1];
              const float* vf = reinterpret_cast<const float*>(v + 8 * q8);
              *reinterpret_cast<uint4*>(orow + c0 + 8 * q8) =
                  make_uint4(pack_bf16x2(vf[0] * f + l0.x, vf[1] * f + l0.y),
                             pack_bf16x2(vf[2] * f + l0.z, vf[3] * f + l0.w),
                             pack_bf16x2(vf[4] * f + l1.x, vf[5] * f + l1.y),
                             pack_bf16x2(vf[6] * f + l1.z, vf[7] * f + l1.w));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <class Kern>
static cudaError_t set_smem(Kern k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_bwd_dq(const CUtensorMap& mapQ, const CUtensorMap& mapdO, const CUtensorMap& mapK,
                          const CUtensorMap& mapV, const BwdSparseArgs& a, int D, int BH,
                          cudaStream_t s) {
  dim3 grid((a.Tq + 1) / 2, BH);
  if (D == 128) {
    const size_t smem = DqSmem<128>::bytes(a.Tkv);
    cudaError_t e = set_smem(bwd_dq_kernel<128>, smem);
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<128><<<grid, 320, smem, s>>>(mapQ, mapdO, mapK, mapV, a);
  } else {
    const size_t smem = DqSmem<64>::bytes(a.Tkv);
    cudaError_t e = set_smem(bwd_dq_kernel<64>, smem);
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<64><<<grid, 320, smem, s>>>(mapQ, mapdO, mapK, mapV, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const CUtensorMap& mapK2, const CUtensorMap& mapV2,
                            const CUtensorMap& mapQ1, const CUtensorMap& mapdO1,
                            const BwdSparseArgs& a, int D, int BH, cudaStream_t s) {
  dim3 grid((a.Tkv + 1) / 2, BH);
  if (D == 128) {
    const size_t smem = DkvSmem<128>::bytes(a.Tq);
    cudaError_t e = set_smem(bwd_dkdv_kernel<128>, smem);
    if (e != cudaSuccess) return e;
    bwd_dkdv_kernel<128><<<grid, 320, smem, s>>>(mapK2, mapV2, mapQ1, mapdO1, a);
  } else {
    const size_t smem = DkvSmem<64>::bytes(a.Tq);
    cudaError_t e = set_smem(bwd_dkdv_kernel<64>, smem);
    if (e != cudaSuccess) return e;
    bwd_dkdv_kernel<64><<<grid, 320, smem, s>>>(mapK2, mapV2, mapQ1, mapdO1, a);
  }
  return cudaGetLastError();
}

}  // namespace sla
