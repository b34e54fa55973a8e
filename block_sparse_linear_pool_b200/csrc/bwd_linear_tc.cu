// Query side of the linear-branch backward on the tensor cores (d = 128).
// Same quantities as bwd_rows_kernel (see bwd_linear.cu for the formulas);
// here a CTA takes query blocks 2p and 2p+1 (128 rows, one TMEM lane each) and
// the three products run as tcgen05.mma:
//   G1  NUM_t  = phi(Q) H'_t           M = 128 rows, N = d, K = d   (t = 0, 1)
//   G2  dphi_t = gp H'_t^T             M = 128 rows, N = d, K = d
//   G3  dH'_t^T = gp_t^T phi(Q_t)      M = d, N = d, K = 64 rows of block t
// G1 and G2 are computed for all 128 rows against both blocks' H' (each row
// keeps the half of its own block), so every per-row scalar (den, o'_r . dO_r,
// D_r) stays with the thread that owns the row.  H'_t arrives by TMA as the
// forward's [H_i^T | Z_i] row ([o][a], a contiguous): the K-major B operand of
// G1 and, read the other way, the MN-major B operand of G2.
//
//   warp 0      TMA: both blocks' H' tiles and Z rows
//   warp 1      tcgen05.mma issuer
//   warps 2-5   one row each: phi(q) -> shared (bf16, swizzled), den; then o',
//               D, gp -> shared, gden; then dq (linear part); finally one row
//               o of dH'_t^T each (G3's lanes are o; the output is [o][a]) and
//               dZ_t[a] for a = its row
// TMEM (512 columns, one CTA per SM): G1 and then G2 at [0, 2d), G3 at [2d, 4d).
#include "kernels.cuh"

namespace sla {

namespace {
constexpr int TD = 128;                       // d
constexpr int TILE = TD * 128;                // one [128 rows][128 B] chunk
constexpr int OFF_H = 0;                      // [2 a-chunks][2 blocks][TD o][128 B]
constexpr int OFF_F = OFF_H + 4 * TILE;       // phi(Q): [2 a-chunks][128 rows][128 B]
constexpr int OFF_G = OFF_F + 2 * TILE;       // gp:     [2 o-chunks][128 rows][128 B]
constexpr int OFF_Z = OFF_G + 2 * TILE;       // Z_t: [2][TD] bf16
constexpr int OFF_GD = OFF_Z + 2 * TD * 2;    // gden [128] fp32
constexpr int OFF_PHI = OFF_GD + 128 * 4;     // phi(q) fp32 [128 rows][TD + 1]
constexpr int OFF_BAR = OFF_PHI + 128 * (TD + 1) * 4;
constexpr int SMEM_TC = OFF_BAR + 256 + 1024;
constexpr float LOG2E_T = 1.4426950408889634f;

__device__ __forceinline__ float bfv(uint32_t packed, int hi) {
  return __uint_as_float(hi ? (packed & 0xffff0000u) : (packed << 16));
}
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
}  // namespace

__global__ void __launch_bounds__(192, 1)
    bwd_rows_tc_kernel(const __grid_constant__ CUtensorMap mapH, const __grid_constant__ CUtensorMap mapZ,
                       BwdRowsArgs a, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sH = sm + OFF_H;
  uint8_t* sF = sm + OFF_F;
  uint8_t* sG = sm + OFF_G;
  const __nv_bfloat16* sZ = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_Z);
  float* sgden = reinterpret_cast<float*>(sm + OFF_GD);
  float* sphi = reinterpret_cast<float*>(sm + OFF_PHI);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* h_full = bars + 0;
  uint64_t* fq_ready = bars + 1;
  uint64_t* num_full = bars + 2;
  uint64_t* gp_ready = bars + 3;
  uint64_t* dphi_full = bars + 4;
  uint64_t* dh_full = bars + 5;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 6);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int i0 = 2 * p, i1 = 2 * p + 1;
  const bool has1 = i1 < a.Tq;

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(h_full, 1);
    mbar_init(fq_ready, 128);
    mbar_init(num_full, 1);
    mbar_init(gp_ready, 128);
    mbar_init(dphi_full, 1);
    mbar_init(dh_full, 1);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (w == 0) {
    if (ln == 0) {
      tma_prefetch_desc(&mapH);
      tma_prefetch_desc(&mapZ);
      mbar_arrive_expect_tx(h_full, 2 * (2 * TILE + TD * 2));
      for (int t = 0; t < 2; ++t) {
        const int i = (t == 1 && has1) ? i1 : i0;  // a missing second block reuses the first
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(sH + c * 2 * TILE + t * TILE, &mapH, h_full, c * 64, 0, i, bh);
          tma_load_3d(sm + OFF_Z + t * TD * 2 + c * 128, &mapZ, h_full, TD * TD + c * 64, i, bh);
        }
      }
    }
  } else if (w == 1) {
    if (ln == 0) {
      const uint32_t id_kk = idesc_bf16(128, TD, false, false);  // A, B K-major
      const uint32_t id_km = idesc_bf16(128, TD, false, true);   // B MN-major
      const uint32_t id_mm = idesc_bf16(128, TD, true, true);    // A, B MN-major
      const uint32_t h0 = smem_u32(sH), f0 = smem_u32(sF), g0 = smem_u32(sG);
      bool ok = mbar_wait(h_full, 0, err, DEV_TIMEOUT_TMA) && mbar_wait(fq_ready, 0, err, DEV_TIMEOUT_SYNC);
      if (ok) {
        tc_fence_after();
        // G1: NUM_t[r][o] = sum_a F[r][a] H'_t[a][o]   (B rows o, K = a contiguous)
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + TD * t, sdesc_sw128(f0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(h0 + (kk / 4) * 2 * TILE + t * TILE + (kk % 4) * 32, 16, 1024), id_kk,
                    kk > 0 ? 1u : 0u);
        umma_commit(num_full);
        ok = mbar_wait(gp_ready, 0, err, DEV_TIMEOUT_SYNC);
      }
      if (ok) {
        tc_fence_after();
        // G2: dphi_t[r][a] = sum_o GP[r][o] H'_t[a][o]   (B: N = a contiguous, K = o rows)
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + TD * t, sdesc_sw128(g0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(h0 + t * TILE + kk * 2048, 2 * TILE, 1024), id_km, kk > 0 ? 1u : 0u);
        umma_commit(dphi_full);
        // G3, transposed: dH'_t^T[o][a] = sum_{r in block t} GP[r][o] F[r][a]  (A: M = o contiguous;
        // B: N = a contiguous), so that a TMEM lane holds one row o of the [o][a] output
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tbase + 2 * TD + TD * t, sdesc_sw128(g0 + t * 8192 + kk * 2048, TILE, 1024),
                    sdesc_sw128(f0 + t * 8192 + kk * 2048, TILE, 1024), id_mm, kk > 0 ? 1u : 0u);
        umma_commit(dh_full);
      }
    }
  } else {
    const int q4 = w & 3;
    const int r = 32 * q4 + ln;          // row (and, for G3, the column a)
    const int t = r >> 6;                // block of this row
    const int i = t == 0 ? i0 : i1;
    const int n = 64 * i + (r & 63);
    const bool valid = (t == 0 || has1) && n < a.N;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    const float cs = a.combine == 1 ? a.alpha[bh] : 1.f;
    const float cl = a.combine == 1 ? 1.f - a.alpha[bh] : 1.f;
    const __nv_bfloat16* qrow = a.Q + (int64_t)b * a.sq[0] + (int64_t)h * a.sq[1] + (int64_t)n * a.sq[2];
    const __nv_bfloat16* drow = a.dO + (int64_t)b * a.so[0] + (int64_t)h * a.so[1] + (int64_t)n * a.so[2];
    const float* osrow = a.os + ((int64_t)bh * a.N + n) * TD;
    if (valid) {  // phase 2's rows into L2 while phase 1 runs
#pragma unroll
      for (int c = 0; c < TD; c += 64) prefetch_l2(drow + c);
#pragma unroll
      for (int c = 0; c < TD; c += 32) prefetch_l2(osrow + c);
    }
    // ---- phase 1: phi(q) (bf16) into sF, den = phi(q) . Z_t + eps.  The row is
    // loaded once, all 16 loads in flight, and kept in registers; the H' and Z
    // tiles are waited for only where den needs Z.
    uint4 qv[TD / 8];
#pragma unroll
    for (int c = 0; c < TD / 8; ++c)
      qv[c] = valid ? __ldg(reinterpret_cast<const uint4*>(qrow) + c) : make_uint4(0u, 0u, 0u, 0u);
    // softmax phi: the row maximum in four partial maxima, then 2^((x - m) log2 e)
    // once per element, kept in sphi until it is normalised below, with the row
    // sum in four partial sums
    float* myphi = sphi + r * (TD + 1);
    float m = -INFINITY, s = 0.f;
    if (valid && a.phi == 0) {
      float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < TD / 8; ++c) {
        const uint32_t u[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) mp[e] = fmax3(mp[e], bfv(u[e], 0), bfv(u[e], 1));
      }
      m = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
      float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < TD / 8; ++c) {
        const uint32_t u[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float e0 = ex2a((bfv(u[e], 0) - m) * LOG2E_T), e1 = ex2a((bfv(u[e], 1) - m) * LOG2E_T);
          myphi[8 * c + 2 * e] = e0;
          myphi[8 * c + 2 * e + 1] = e1;
          sp[e] += e0 + e1;
        }
      }
      s = (sp[0] + sp[1]) + (sp[2] + sp[3]);
    }
    const float inv_s = (a.phi == 0 && s > 0.f) ? 1.f / s : 1.f;
    auto phi_at = [&](int col, float x) {
      return a.phi == 1 ? (x > 0.f ? x + 1.f : ex2a(x * LOG2E_T)) : myphi[col] * inv_s;
    };
    float den = a.eps;
    bool ok = __all_sync(0xffffffffu, mbar_wait(h_full, 0, err, DEV_TIMEOUT_TMA));
    if (ok) {
      const __nv_bfloat16* z = sZ + t * TD;
      float dp[4] = {0.f, 0.f, 0.f, 0.f};  // den in four partial sums
#pragma unroll
      for (int c = 0; c < TD; c += 8) {
        uint32_t o4[4] = {0u, 0u, 0u, 0u};
        if (valid) {
          const uint4 v = qv[c / 8];
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float f0 = phi_at(c + 2 * e, bfv(u[e], 0)), f1 = phi_at(c + 2 * e + 1, bfv(u[e], 1));
            myphi[c + 2 * e] = f0;
            myphi[c + 2 * e + 1] = f1;
            o4[e] = pack_bf16x2(f0, f1);
            dp[e] = fmaf(bfv(o4[e], 0), __bfloat162float(z[c + 2 * e]),
                         fmaf(bfv(o4[e], 1), __bfloat162float(z[c + 2 * e + 1]), dp[e]));
          }
        }
        *reinterpret_cast<uint4*>(sF + (c / 64) * TILE + sw128_offset(r, (c % 64) * 2)) =
            make_uint4(o4[0], o4[1], o4[2], o4[3]);
      }
      den += (dp[0] + dp[1]) + (dp[2] + dp[3]);
    }
    fence_proxy_async_smem();
    mbar_arrive(fq_ready);
    // ---- phase 2: o' = NUM / den, D, gp (bf16) into sG, gden
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(num_full, 0, err, DEV_TIMEOUT_MMA));
    float dd = 0.f, dol = 0.f, da = 0.f;
    if (ok) {
      tc_fence_after();
      const float inv_den = 1.f / den;
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        // this chunk's dO and o^s loads go out before the TMEM load, all in flight
        uint4 dq4[4];
        float4 os4[8];
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          dq4[v4] = valid ? __ldg(reinterpret_cast<const uint4*>(drow + c0) + v4) : make_uint4(0u, 0u, 0u, 0u);
          os4[2 * v4] = valid ? __ldg(reinterpret_cast<const float4*>(osrow + c0) + 2 * v4) : make_float4(0.f, 0.f, 0.f, 0.f);
          os4[2 * v4 + 1] = valid ? __ldg(reinterpret_cast<const float4*>(osrow + c0) + 2 * v4 + 1)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t nv[32];
        tmem_ld32(tl + TD * t + c0, nv);
        tmem_ld_wait();
        uint32_t gpk[16];
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) {
          float dov[8], osv[8];
          {
            const uint4 v = dq4[c8 / 8];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) dov[e] = bfv(u[e / 2], e & 1);
            const float4 o0 = os4[c8 / 4], o1 = os4[c8 / 4 + 1];
            osv[0] = o0.x; osv[1] = o0.y; osv[2] = o0.z; osv[3] = o0.w;
            osv[4] = o1.x; osv[5] = o1.y; osv[6] = o1.z; osv[7] = o1.w;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float ol = __uint_as_float(nv[c8 + e]) * inv_den;  // o'_r
            dd = fmaf(cs * dov[e], osv[e], dd);
            dol = fmaf(dov[e], ol, dol);
            da = fmaf(osv[e] - ol, dov[e], da);
          }
#pragma unroll
          for (int e = 0; e < 8; e += 2)
            gpk[(c8 + e) / 2] = pack_bf16x2(cl * dov[e] * inv_den, cl * dov[e + 1] * inv_den);
        }
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          *reinterpret_cast<uint4*>(sG + (c0 / 64) * TILE + sw128_offset(r, ((c0 % 64) + 8 * v4) * 2)) =
              make_uint4(gpk[4 * v4], gpk[4 * v4 + 1], gpk[4 * v4 + 2], gpk[4 * v4 + 3]);
      }
    }
    const float gden = valid ? -cl * dol / den : 0.f;
    sgden[r] = gden;
    if (valid) a.ld2[(int64_t)bh * a.Tq * 64 + n] = make_float2(-a.lse[(int64_t)bh * a.N + n] * LOG2E_T, -dd);
    else if (t == 0 || has1) a.ld2[(int64_t)bh * a.Tq * 64 + n] = make_float2(-INFINITY, 0.f);
    if (a.combine == 1 && a.dalpha) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
      if (ln == 0) atomicAdd(a.dalpha + bh, da);
    }
    fence_proxy_async_smem();
    mbar_arrive(gp_ready);
    // ---- phase 3: dq (linear part) = phi backward of dphi = G2 + gden Z_t
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dphi_full, 0, err, DEV_TIMEOUT_MMA));
    if (ok) {
      tc_fence_after();
      const __nv_bfloat16* z = sZ + t * TD;
      float dot = 0.f;
      if (a.phi == 0) {
        float dq4[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums
#pragma unroll 1
        for (int c0 = 0; c0 < TD; c0 += 32) {
          uint32_t dv[32];
          tmem_ld32(tl + TD * t + c0, dv);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              dq4[e & 3] = fmaf(myphi[c0 + e], __uint_as_float(dv[e]) + gden * __bfloat162float(z[c0 + e]),
                                dq4[e & 3]);
          }
        }
        dot = (dq4[0] + dq4[1]) + (dq4[2] + dq4[3]);
      }
      float* out = a.dq_lin + ((int64_t)bh * a.N + n) * TD;
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        uint32_t dv[32];
        tmem_ld32(tl + TD * t + c0, dv);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e4 = 0; e4 < 32; e4 += 4) {
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float f = myphi[c0 + e4 + e];
              const float dphi = __uint_as_float(dv[e4 + e]) + gden * __bfloat162float(z[c0 + e4 + e]);
              // elu + 1: d phi / dx = 1 where x > 0 (phi > 1), else e^x = phi
              y[e] = a.phi == 1 ? dphi * (f > 1.f ? 1.f : f) : f * (dphi - dot);
            }
            *reinterpret_cast<float4*>(out + c0 + e4) = make_float4(y[0], y[1], y[2], y[3]);
          }
        }
      }
    }
    // ---- phase 4: thread r owns row o = r of dH'_t^T (G3's lanes: the [o][a] row
    // of the output, 16-byte stores) and dZ_t[a = r]; the waits on fq_ready /
    // gp_ready order the other rows' phi(q) and gden writes
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dh_full, 0, err, DEV_TIMEOUT_MMA) &&
                                             mbar_wait(fq_ready, 0, err, DEV_TIMEOUT_SYNC) &&
                                             mbar_wait(gp_ready, 0, err, DEV_TIMEOUT_SYNC));
    if (ok) {
      tc_fence_after();
      const int aa = r;
      for (int tt = 0; tt < (has1 ? 2 : 1); ++tt) {
        const int it = tt == 0 ? i0 : i1;
        __nv_bfloat16* dst = a.dhz + ((int64_t)bh * a.Tq + it) * a.NN;
#pragma unroll 1
        for (int c0 = 0; c0 < TD; c0 += 32) {
          uint32_t hv[32];
          tmem_ld32(tl + 2 * TD + TD * tt + c0, hv);
          tmem_ld_wait();
          uint4* d4 = reinterpret_cast<uint4*>(dst + (int64_t)aa * TD + c0);  // row o = aa, a = c0 ..
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(
                pack_bf16x2(__uint_as_float(hv[8 * v4]), __uint_as_float(hv[8 * v4 + 1])),
                pack_bf16x2(__uint_as_float(hv[8 * v4 + 2]), __uint_as_float(hv[8 * v4 + 3])),
                pack_bf16x2(__uint_as_float(hv[8 * v4 + 4]), __uint_as_float(hv[8 * v4 + 5])),
                pack_bf16x2(__uint_as_float(hv[8 * v4 + 6]), __uint_as_float(hv[8 * v4 + 7])));
        }
        // dZ_t[a] = sum_{rows of block tt} gden_r phi(q_r)[a], in eight partial sums
        float dzp[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) dzp[q] = 0.f;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const int rr = 64 * tt + k;
          const __nv_bfloat16* fp = reinterpret_cast<const __nv_bfloat16*>(
              sF + (aa / 64) * TILE + sw128_offset(rr, (aa % 64) * 2));
          dzp[k & 7] = fmaf(sgden[rr], __bfloat162float(*fp), dzp[k & 7]);
        }
        const float dz = ((dzp[0] + dzp[1]) + (dzp[2] + dzp[3])) + ((dzp[4] + dzp[5]) + (dzp[6] + dzp[7]));
        dst[TD * TD + aa] = __float2bfloat16(dz);
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

cudaError_t launch_bwd_rows_tc(const CUtensorMap& mapH, const CUtensorMap& mapZ, const BwdRowsArgs& a,
                               int* err, int BH, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_rows_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_TC);
  if (e != cudaSuccess) return e;
  bwd_rows_tc_kernel<<<dim3((a.Tq + 1) / 2, BH), 192, SMEM_TC, s>>>(mapH, mapZ, a, err);
  return cudaGetLastError();
}

// Column sums of dO over every row of every head (d bias of Proj).  256
// threads = 16 row lanes x 16 groups of 8 columns (16-byte loads); a CTA sums
// 1024 rows, reduces its 16 row lanes in shared memory and adds one atomic per
// column.
__global__ void __launch_bounds__(256) colsum_kernel(const __nv_bfloat16* __restrict__ dO, const int64_t s0,
                                                     const int64_t s1, const int64_t s2, int H, int N,
                                                     int64_t rows, float* __restrict__ out) {
  __shared__ float red[16][TD + 4];
  const int cg = threadIdx.x & 15, rl = threadIdx.x >> 4;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int64_t r0 = (int64_t)blockIdx.x * 1024;
  for (int64_t r = r0 + rl; r < min(r0 + 1024, rows); r += 16) {
    const int64_t bh = r / N, n = r % N;
    const uint4 v = *reinterpret_cast<const uint4*>(dO + (bh / H) * s0 + (bh % H) * s1 + n * s2 + 8 * cg);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += bfv(u[e / 2], e & 1);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rl][8 * cg + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < TD) {
    float t = 0.f;
    for (int k = 0; k < 16; ++k) t += red[k][threadIdx.x];
    atomicAdd(out + threadIdx.x, t);
  }
}

cudaError_t launch_colsum(const __nv_bfloat16* dO, const int64_t* so, int H, int N, int BH, int D,
                          float* out, cudaStream_t s) {
  if (D != TD) return cudaErrorInvalidValue;
  const int64_t rows = (int64_t)BH * N;
  colsum_kernel<<<(unsigned)((rows + 1023) / 1024), 256, 0, s>>>(dO, so[0], so[1], so[2], H, N, rows, out);
  return cudaGetLastError();
}

}  // namespace sla

namespace sla {

// ---------------------------------------------------------------------------
// Key side of the linear-branch backward on the tensor cores (d = 128).  A CTA
// takes key blocks 2p and 2p+1 (128 key rows, one TMEM lane each):
//   G1  U_t    = phi(K) dh'_t          M = 128 rows, N = d, K = d  (t = 0, 1)
//   G3  w      = V W~^T                M = 128 rows, N = d, K = d  (SLA; w = V for SLA2)
//   G2  dv     = U W~                  M = 128 rows, N = d, K = d  (SLA; dv = U for SLA2)
//   G4  dphi_t = w dh'_t^T             M = 128 rows, N = d, K = d
// then dk = phi backward of dphi + dz.  dW = sum_t u_t v_t^T is left to
// dw_kernel: U (bf16, rows of every head) goes to a buffer.
// TMEM (512 columns): G1 and then G4 at [0, 2d), G3 and then G2 at [2d, 3d),
// phi(K) in fp32 at [3d, 4d).
// ---------------------------------------------------------------------------
namespace {
constexpr int K_OFF_G = 0;                     // dh': [2 a-chunks][2 blocks][TD o][128 B]
constexpr int K_OFF_F = K_OFF_G + 4 * TILE;    // phi(K), then w: [2 chunks][128 rows][128 B]
constexpr int K_OFF_V = K_OFF_F + 2 * TILE;    // V pair
constexpr int K_OFF_U = K_OFF_V + 2 * TILE;    // U (bf16)
constexpr int K_OFF_W = K_OFF_U + 2 * TILE;    // W~ (bf16): [2 c-chunks][TD o][128 B]
constexpr int K_OFF_Z = K_OFF_W + 2 * TILE;    // dz_t: [2][TD] bf16
constexpr int K_OFF_BAR = K_OFF_Z + 2 * TD * 2;
constexpr int K_SMEM = K_OFF_BAR + 256 + 1024;
}  // namespace

__global__ void __launch_bounds__(192, 1)
    bwd_keys_tc_kernel(const __grid_constant__ CUtensorMap mapG, const __grid_constant__ CUtensorMap mapZ,
                       const __grid_constant__ CUtensorMap mapK2, const __grid_constant__ CUtensorMap mapV2,
                       BwdKeysArgs a, __nv_bfloat16* ubuf, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sG = sm + K_OFF_G;
  uint8_t* sF = sm + K_OFF_F;
  uint8_t* sV = sm + K_OFF_V;
  uint8_t* sU = sm + K_OFF_U;
  uint8_t* sW = sm + K_OFF_W;
  const __nv_bfloat16* sZ = reinterpret_cast<const __nv_bfloat16*>(sm + K_OFF_Z);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + K_OFF_BAR);
  uint64_t* in_full = bars + 0;   // dh' tiles, Z rows, V pair
  uint64_t* fk_ready = bars + 1;
  uint64_t* g1_full = bars + 2;
  uint64_t* u_ready = bars + 3;
  uint64_t* g2_full = bars + 4;
  uint64_t* k_full = bars + 5;    // K pair: phi(K) starts while the rest is loading
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 6);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int j0 = 2 * p, j1 = 2 * p + 1;
  const bool has1 = j1 < a.Tkv;
  const bool proj = a.proj_w != nullptr;

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(in_full, 1);
    mbar_init(fk_ready, 128);
    mbar_init(g1_full, 1);
    mbar_init(u_ready, 128);
    mbar_init(g2_full, 1);
    mbar_init(k_full, 1);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (w == 0) {
    if (ln == 0) {
      tma_prefetch_desc(&mapG);
      tma_prefetch_desc(&mapZ);
      tma_prefetch_desc(&mapK2);
      tma_prefetch_desc(&mapV2);
      mbar_arrive_expect_tx(k_full, 2 * TILE);
#pragma unroll
      for (int c = 0; c < 2; ++c) tma_load_4d(sF + c * TILE, &mapK2, k_full, c * 64, 128 * p, h, b);
      mbar_arrive_expect_tx(in_full, 2 * (2 * TILE + TD * 2) + 2 * TILE);
      for (int t = 0; t < 2; ++t) {
        const int j = (t == 1 && has1) ? j1 : j0;  // a missing second block reuses the first
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(sG + c * 2 * TILE + t * TILE, &mapG, in_full, c * 64, 0, j, bh);
          tma_load_3d(sm + K_OFF_Z + t * TD * 2 + c * 128, &mapZ, in_full, TD * TD + c * 64, j, bh);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) tma_load_4d(sV + c * TILE, &mapV2, in_full, c * 64, 128 * p, h, b);
    }
  } else if (w == 1) {
    if (ln == 0) {
      const uint32_t id_kk = idesc_bf16(128, TD, false, false);
      const uint32_t id_km = idesc_bf16(128, TD, false, true);
      const uint32_t g0 = smem_u32(sG), f0 = smem_u32(sF), v0 = smem_u32(sV), u0 = smem_u32(sU),
                     w0 = smem_u32(sW);
      bool ok = mbar_wait(in_full, 0, err, DEV_TIMEOUT_TMA) && mbar_wait(fk_ready, 0, err, DEV_TIMEOUT_SYNC);
      if (ok) {
        tc_fence_after();
        // G1: U_t[r][o] = sum_a F[r][a] dh'_t[a][o]
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + TD * t, sdesc_sw128(f0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(g0 + (kk / 4) * 2 * TILE + t * TILE + (kk % 4) * 32, 16, 1024), id_kk,
                    kk > 0 ? 1u : 0u);
        // G3: w[r][o] = sum_c V[r][c] W[o][c]
        if (proj)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + 2 * TD, sdesc_sw128(v0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(w0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        umma_commit(g1_full);
        ok = mbar_wait(u_ready, 0, err, DEV_TIMEOUT_SYNC);
      }
      if (ok) {
        tc_fence_after();
        // G2: dv[r][c] = sum_o U[r][o] W[o][c]   (B: N = c contiguous, K = o rows)
        if (proj)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + 2 * TD, sdesc_sw128(u0 + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(w0 + kk * 2048, TILE, 1024), id_km, kk > 0 ? 1u : 0u);
        // G4: dphi_t[r][a] = sum_o w[r][o] dh'_t[a][o]   (w in sF for SLA, V itself for SLA2)
        const uint32_t ws = proj ? f0 : v0;
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int kk = 0; kk < TD / 16; ++kk)
            umma_ss(tbase + TD * t, sdesc_sw128(ws + (kk / 4) * TILE + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(g0 + t * TILE + kk * 2048, 2 * TILE, 1024), id_km, kk > 0 ? 1u : 0u);
        umma_commit(g2_full);
      }
    }
  } else {
    const int q4 = w & 3;
    const int r = 32 * q4 + ln;  // key row of the pair
    const int t = r >> 6;
    const int n = 128 * p + r;
    const bool valid = (t == 0 || has1) && n < a.N;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    // W~ as bf16 into sW (row o = r), the K-major B operand of G3 / MN-major B of G2
    if (proj) {  // the whole row's loads in flight at once
      const float4* wr4 = reinterpret_cast<const float4*>(a.proj_w + (int64_t)r * TD);
      float4 x[TD / 4];
#pragma unroll
      for (int c = 0; c < TD / 4; ++c) x[c] = __ldg(wr4 + c);
#pragma unroll
      for (int c = 0; c < TD; c += 8) {
        const float4 x0 = x[c / 4], x1 = x[c / 4 + 1];
        *reinterpret_cast<uint4*>(sW + (c / 64) * TILE + sw128_offset(r, (c % 64) * 2)) =
            make_uint4(pack_bf16x2(x0.x, x0.y), pack_bf16x2(x0.z, x0.w), pack_bf16x2(x1.x, x1.y),
                       pack_bf16x2(x1.z, x1.w));
      }
    }
    bool ok = __all_sync(0xffffffffu, mbar_wait(k_full, 0, err, DEV_TIMEOUT_TMA));
    // ---- phi(K) in place (bf16); rows that do not exist get 0
    float m = -INFINITY, s = 0.f;
    if (ok && valid && a.phi == 0) {  // from the K tile in shared memory (loaded by TMA)
      uint4 kv[TD / 8];
#pragma unroll
      for (int c = 0; c < TD / 8; ++c)
        kv[c] = *reinterpret_cast<const uint4*>(sF + (c / 8) * TILE + sw128_offset(r, (c % 8) * 16));
      // the row maximum and sum in four partial maxima / sums each
      float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < TD / 8; ++c) {
        const uint32_t u[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) mp[e] = fmax3(mp[e], bfv(u[e], 0), bfv(u[e], 1));
      }
      m = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
      float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < TD / 8; ++c) {
        const uint32_t u[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sp[e] += ex2a((bfv(u[e], 0) - m) * LOG2E_T) + ex2a((bfv(u[e], 1) - m) * LOG2E_T);
      }
      s = (sp[0] + sp[1]) + (sp[2] + sp[3]);
    }
    const float inv_s = (a.phi == 0 && s > 0.f) ? 1.f / s : 1.f;
    auto phi_of = [&](float x) {
      return a.phi == 1 ? (x > 0.f ? x + 1.f : ex2a(x * LOG2E_T)) : ex2a((x - m) * LOG2E_T) * inv_s;
    };
    // phi(K) in place in sF (bf16, the MMA operand) and in fp32 in TMEM columns
    // [3d, 4d) of this row's lane, for the phi backward at the end
    if (ok) {
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        uint32_t fv[32];
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) {
          uint8_t* dst = sF + (c0 / 64) * TILE + sw128_offset(r, ((c0 % 64) + c8) * 2);
          uint32_t o4[4] = {0u, 0u, 0u, 0u};
          if (valid) {
            const uint4 v = *reinterpret_cast<const uint4*>(dst);  // K as loaded (bf16)
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float f0 = phi_of(bfv(u[e], 0)), f1 = phi_of(bfv(u[e], 1));
              fv[c8 + 2 * e] = __float_as_uint(f0);
              fv[c8 + 2 * e + 1] = __float_as_uint(f1);
              o4[e] = pack_bf16x2(f0, f1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) fv[c8 + e] = 0u;
          }
          *reinterpret_cast<uint4*>(dst) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        tmem_st32(tl + 3 * TD + c0, fv);
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    mbar_arrive(fk_ready);
    // ---- U (own block's half) -> sU (and the U buffer for dW, SLA); dv = U for SLA2;
    //      w -> sF (SLA)
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(g1_full, 0, err, DEV_TIMEOUT_MMA));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* urow = ubuf ? ubuf + ((int64_t)bh * a.Tkv * 64 + n) * TD : nullptr;
      float* dvrow = a.dv_lin + ((int64_t)bh * a.N + n) * TD;
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        uint32_t uv[32];
        tmem_ld32(tl + TD * t + c0, uv);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = valid ? pack_bf16x2(__uint_as_float(uv[2 * e]), __uint_as_float(uv[2 * e + 1])) : 0u;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint4 q = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          *reinterpret_cast<uint4*>(sU + (c0 / 64) * TILE + sw128_offset(r, ((c0 % 64) + 8 * v4) * 2)) = q;
          if (urow && (t == 0 || has1) && n < a.Tkv * 64) reinterpret_cast<uint4*>(urow + c0)[v4] = q;
        }
        if (!proj && valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dvrow + c0 + e) =
                make_float4(__uint_as_float(uv[e]), __uint_as_float(uv[e + 1]), __uint_as_float(uv[e + 2]),
                            __uint_as_float(uv[e + 3]));
        }
      }
      if (proj) {
#pragma unroll 1
        for (int c0 = 0; c0 < TD; c0 += 32) {
          uint32_t wv[32];
          tmem_ld32(tl + 2 * TD + c0, wv);
          tmem_ld_wait();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint32_t q[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              q[e] = pack_bf16x2(__uint_as_float(wv[8 * v4 + 2 * e]), __uint_as_float(wv[8 * v4 + 2 * e + 1]));
            *reinterpret_cast<uint4*>(sF + (c0 / 64) * TILE + sw128_offset(r, ((c0 % 64) + 8 * v4) * 2)) =
                make_uint4(q[0], q[1], q[2], q[3]);
          }
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(u_ready);
    // ---- dv (SLA) and dk = phi backward of dphi_t + dz_t.  tcgen05.ld is a
    // warp-wide instruction: every lane runs it, only valid rows store.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(g2_full, 0, err, DEV_TIMEOUT_MMA) &&
                                             mbar_wait(in_full, 0, err, DEV_TIMEOUT_TMA));  // Z rows
    if (ok) {
      tc_fence_after();
      if (proj) {
        float* dvrow = a.dv_lin + ((int64_t)bh * a.N + n) * TD;
#pragma unroll 1
        for (int c0 = 0; c0 < TD; c0 += 32) {
          uint32_t dv[32];
          tmem_ld32(tl + 2 * TD + c0, dv);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dvrow + c0 + e) =
                  make_float4(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1]), __uint_as_float(dv[e + 2]),
                              __uint_as_float(dv[e + 3]));
          }
        }
      }
      const __nv_bfloat16* z = sZ + t * TD;
      float dot = 0.f;
      if (a.phi == 0) {
        float dq4[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums
#pragma unroll 1
        for (int c0 = 0; c0 < TD; c0 += 32) {
          uint32_t dv[32], fv[32];
          tmem_ld32(tl + TD * t + c0, dv);
          tmem_ld32(tl + 3 * TD + c0, fv);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              dq4[e & 3] = fmaf(__uint_as_float(fv[e]), __uint_as_float(dv[e]) + __bfloat162float(z[c0 + e]),
                                dq4[e & 3]);
          }
        }
        dot = (dq4[0] + dq4[1]) + (dq4[2] + dq4[3]);
      }
      float* out = a.dk_lin + ((int64_t)bh * a.N + n) * TD;
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        uint32_t dv[32], fv[32];
        tmem_ld32(tl + TD * t + c0, dv);
        tmem_ld32(tl + 3 * TD + c0, fv);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e4 = 0; e4 < 32; e4 += 4) {
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float f = __uint_as_float(fv[e4 + e]);
              const float dphi = __uint_as_float(dv[e4 + e]) + __bfloat162float(z[c0 + e4 + e]);
              // elu + 1: d phi / dx = 1 where x > 0 (phi > 1), else e^x = phi
              y[e] = a.phi == 1 ? dphi * (f > 1.f ? 1.f : f) : f * (dphi - dot);
            }
            *reinterpret_cast<float4*>(out + c0 + e4) = make_float4(y[0], y[1], y[2], y[3]);
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
// dW = sum over every token row of u_t v_t^T (SLA's Proj weight gradient):
// persistent, CTA c sums 128-row tiles c, c + G, ... of all heads into one
// 128 x 128 TMEM accumulator (A = U^T and B = V, both MN-major: the rows are
// the reduction), then adds it to dproj_w with one atomic per element.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(192, 1)
    dw_kernel(const __grid_constant__ CUtensorMap mapU, const __grid_constant__ CUtensorMap mapV2,
              int H, int Tkv, int ntiles_head, int ntiles, float* __restrict__ dW, int* err) {
  extern __shared__ uint8_t smem_dw[];  // 2 stages of (U tile, V tile), 1024-byte aligned
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dw) + 1023) & ~uintptr_t(1023));
  (void)Tkv;
  __shared__ uint64_t full[2], empty[2], done;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  if (w == 1) {
    tmem_alloc(&tslot, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&full[x], 1);
      mbar_init(&empty[x], 1);
    }
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  int my = 0;
  for (int tt = blockIdx.x; tt < ntiles; tt += gridDim.x) ++my;
  if (w == 0 && ln == 0) {
    bool ok = true;
    int k = 0;
    for (int tt = blockIdx.x; tt < ntiles && ok; tt += gridDim.x, ++k) {
      const int x = k & 1;
      if (k >= 2 && !mbar_wait(&empty[x], ((k - 2) >> 1) & 1, err, DEV_TIMEOUT_SYNC)) { ok = false; break; }
      const int bh = tt / ntiles_head, r0 = 128 * (tt % ntiles_head);
      uint8_t* st = sm + x * 4 * TILE;
      mbar_arrive_expect_tx(&full[x], 4 * TILE);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_3d(st + c * TILE, &mapU, &full[x], c * 64, r0, bh);
        tma_load_4d(st + 2 * TILE + c * TILE, &mapV2, &full[x], c * 64, r0, bh % H, bh / H);
      }
    }
  } else if (w == 1 && ln == 0) {
    const uint32_t id_mm = idesc_bf16(128, TD, true, true);
    bool ok = true;
    for (int k = 0; k < my && ok; ++k) {
      const int x = k & 1;
      if (!mbar_wait(&full[x], (k >> 1) & 1, err, DEV_TIMEOUT_TMA)) { ok = false; break; }
      tc_fence_after();
      const uint32_t st = smem_u32(sm + x * 4 * TILE);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_ss(tbase, sdesc_sw128(st + kk * 2048, TILE, 1024), sdesc_sw128(st + 2 * TILE + kk * 2048, TILE, 1024),
                id_mm, (k > 0 || kk > 0) ? 1u : 0u);
      umma_commit(&empty[x]);
    }
    if (ok) umma_commit(&done);
  } else if (w >= 2) {
    const int q4 = w & 3;
    const int o = 32 * q4 + ln;
    if (my > 0 && __all_sync(0xffffffffu, mbar_wait(&done, 0, err, DEV_TIMEOUT_MMA))) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < TD; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + ((uint32_t)(32 * q4) << 16) + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) atomicAdd(dW + (int64_t)o * TD + c0 + e, __uint_as_float(v[e]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

cudaError_t launch_bwd_keys_tc(const CUtensorMap& mapG, const CUtensorMap& mapZ, const CUtensorMap& mapK2,
                               const CUtensorMap& mapV2, const BwdKeysArgs& a, __nv_bfloat16* ubuf, int* err,
                               cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_keys_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM);
  if (e != cudaSuccess) return e;
  bwd_keys_tc_kernel<<<dim3((a.Tkv + 1) / 2, a.BH), 192, K_SMEM, s>>>(mapG, mapZ, mapK2, mapV2, a, ubuf, err);
  return cudaGetLastError();
}

cudaError_t launch_dw(const CUtensorMap& mapU, const CUtensorMap& mapV2, int H, int BH, int Tkv, float* dW,
                      int* err, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_head = (Tkv * 64 + 127) / 128;
  const int ntiles = per_head * BH;
  const int smem = 2 * 4 * TILE + 1024;
  cudaError_t e = cudaFuncSetAttribute(dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dw_kernel<<<ntiles < sms ? ntiles : sms, 192, smem, s>>>(mapU, mapV2, H, Tkv, per_head, ntiles, dW, err);
  return cudaGetLastError();
}

}  // namespace sla
