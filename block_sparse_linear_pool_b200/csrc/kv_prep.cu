// Per-key-block linear-attention statistics ("SLA: Beyond Sparsity in
// Diffusion Transformers via Fine-Tunable Sparse-Linear Attention", §2 Q2
// step 3 and Fig. 4 "Linear Attention Precomputation"):
//     h_j = phi(K_j)^T V_j,   z_j = rowsum(phi(K_j)^T),   phi = softmax over d
// (or elu + 1, the feature-map ablation of the same page's Table 2).
// With the SLA combine, Proj's weight W is folded in (h_j W^T is stored):
// Proj(O^l) = phi(Q) (H W^T) / den + b because den is a per-row scalar.
//
// One CTA (4 warps, two per SM) walks key blocks of 64 tokens persistently
// through three shared-memory stages, the next two blocks' K_j, V_j loading
// while the current one is processed:
//   TMA      K_j, V_j  -> stage (128B-swizzled, d contiguous)
//   tcgen05  D1 = W V_j^T          (M = d, N = 64, K = d)   [SLA only; for
//            d = 128 W is the A operand from TMEM, which leaves the shared
//            memory to the three stages]
//   threads  phi(K_j) in place of K_j; V'^T = D1 in place of V_j (bf16)
//   tcgen05  D2 = V'^T phi(K_j)    (M = d, N = d, K = 64)  = (h_j W^T)^T
//   threads  z_j = column sums of phi(K_j); D2 -> the stage as a swizzled
//            d x d tile, then one TMA store writes it to hz (coalesced)
#include "kernels.cuh"

namespace sla {

template <int D>
struct KvSmem {
  static constexpr int CH = D / 64;                 // 64-column chunks of d
  static constexpr bool W_TMEM = D == 128;          // W in TMEM columns [192, 256) as bf16 pairs
  static constexpr int W_BYTES = W_TMEM ? 0 : D * D * 2;  // else W, K-major [CH][D rows][128B]
  static constexpr int T_BYTES = 64 * D * 2;        // one 64-token tile
  static constexpr int STAGE = 2 * T_BYTES;         // K (then phi) | V (then V'^T); then the h tile
  static constexpr int NST = 3;                     // stages
  static constexpr int OFF_W = 0;
  static constexpr int OFF_ST = OFF_W + W_BYTES;
  static constexpr int OFF_BAR = OFF_ST + NST * STAGE;
  static constexpr int BYTES = OFF_BAR + 64;
  static constexpr int ALLOC = BYTES + 1024;        // slack for 1024-byte alignment
};
static_assert(KvSmem<128>::STAGE >= 128 * 128 * 2 && KvSmem<64>::STAGE >= 64 * 64 * 2,
              "the h tile must fit one stage");

template <int D>
__global__ void __launch_bounds__(128) kv_prep_kernel(const __grid_constant__ CUtensorMap mapK,
                                                      const __grid_constant__ CUtensorMap mapV,
                                                      const __grid_constant__ CUtensorMap mapO,
                                                      KvPrepArgs a) {
  using L = KvSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sW = sm + L::OFF_W;
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);  // [NST]
  uint64_t* mma_bar = tma_bar + L::NST;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mma_bar + 1);
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const bool proj = a.proj_w != nullptr;

  if (w == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int x = 0; x < L::NST; ++x) mbar_init(&tma_bar[x], 1);
    mbar_init(mma_bar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    tma_prefetch_desc(&mapO);
  }
  if (proj && !L::W_TMEM) {  // W (fp32 [o][b]) -> bf16, K-major over b
    for (int g = tid; g < D * D / 8; g += 128) {
      const int o = g / (D / 8), b0 = (g % (D / 8)) * 8;
      const float4 x0 = __ldg(reinterpret_cast<const float4*>(a.proj_w + o * D + b0));
      const float4 x1 = __ldg(reinterpret_cast<const float4*>(a.proj_w + o * D + b0 + 4));
      uint4 v;
      v.x = pack_bf16x2(x0.x, x0.y);
      v.y = pack_bf16x2(x0.z, x0.w);
      v.z = pack_bf16x2(x1.x, x1.y);
      v.w = pack_bf16x2(x1.z, x1.w);
      *reinterpret_cast<uint4*>(sW + (b0 / 64) * (D * 128) + sw128_offset(o, (b0 % 64) * 2)) = v;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t tD1 = tbase;       // 64 columns
  const uint32_t tD2 = tbase + 64;  // D columns
  const uint32_t tW = tbase + 192;  // d = 128: W, row o in lane o, bf16 pairs along b
  const uint32_t lane_off = (uint32_t)(32 * (w & 3)) << 16;
  if (proj && L::W_TMEM) {  // thread tid holds row o = tid (lane tid)
    const float* wr = a.proj_w + (int64_t)tid * D;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 x0 = __ldg(reinterpret_cast<const float4*>(wr + 64 * half + 8 * c));
        const float4 x1 = __ldg(reinterpret_cast<const float4*>(wr + 64 * half + 8 * c + 4));
        r[4 * c + 0] = pack_bf16x2(x0.x, x0.y);
        r[4 * c + 1] = pack_bf16x2(x0.z, x0.w);
        r[4 * c + 2] = pack_bf16x2(x1.x, x1.y);
        r[4 * c + 3] = pack_bf16x2(x1.z, x1.w);
      }
      tmem_st32(tW + lane_off + 32 * half, r);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // Row of the M = D accumulators held by this thread (M = 64 packs rows
  // 16 per 32-lane quarter).
  const int my_row = (D == 128) ? tid : ((ln < 16) ? 16 * w + ln : -1);

  auto issue_load = [&](int item, int s) {
    const int bh = item / a.Tkv, j = item % a.Tkv;
    const int b = bh / a.H, h = bh % a.H;
    uint8_t* st = sm + L::OFF_ST + s * L::STAGE;
    mbar_arrive_expect_tx(&tma_bar[s], 2 * L::T_BYTES);
#pragma unroll
    for (int c = 0; c < L::CH; ++c) {
      tma_load_4d(st + c * 8192, &mapK, &tma_bar[s], c * 64, j * 64, h, b);
      tma_load_4d(st + L::T_BYTES + c * 8192, &mapV, &tma_bar[s], c * 64, j * 64, h, b);
    }
  };
  int n_issued = 0;  // loads issued (thread 0)
  if (tid == 0) {
    for (int x = 0; x < L::NST - 1; ++x)
      if ((int)blockIdx.x + x * (int)gridDim.x < a.nitems) {
        issue_load(blockIdx.x + x * gridDim.x, x);
        ++n_issued;
      }
  }

  uint32_t mma_phase = 0;
  int n = 0;
  // Every wait result is agreed on by the whole CTA (__syncthreads_and), so a
  // timeout makes all threads leave the loop at the same point.
  for (int item = blockIdx.x; item < a.nitems; item += gridDim.x, ++n) {
    const int s = n % L::NST;
    uint8_t* sK = sm + L::OFF_ST + s * L::STAGE;
    uint8_t* sV = sK + L::T_BYTES;
    const int bh = item / a.Tkv, j = item % a.Tkv;
    const int cnt = min(64, a.N - j * 64);
    if (!__syncthreads_and(mbar_wait(&tma_bar[s], (n / L::NST) & 1, a.err, DEV_TIMEOUT_TMA))) break;
    if (proj && tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(D, 64, false, false);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k % 4) * 32;
        const uint64_t bd = sdesc_sw128(smem_u32(sV) + (k / 4) * 8192 + off, 16, 1024);
        if (L::W_TMEM) {  // b = 16 k .. 16 k + 15: columns 8 k .. 8 k + 7 of W
          umma_ts(tD1, tW + 8 * k, bd, id, k > 0);
        } else {
          const uint64_t ad = sdesc_sw128(smem_u32(sW) + (k / 4) * (D * 128) + off, 16, 1024);
          umma_ss(tD1, ad, bd, id, k > 0);
        }
      }
      umma_commit(mma_bar);
    }
    {  // phi(K_j) in place: two threads per token row, each owning D/2 columns.
      constexpr int NE = D / 2;
      const int t = tid >> 1, half = tid & 1;
      const int chunk = (D == 128) ? half : 0;
      const int byte0 = (D == 128) ? 0 : half * 64;
      float x[NE];
#pragma unroll
      for (int v = 0; v < NE / 8; ++v) {
        const uint4 q = *reinterpret_cast<const uint4*>(sK + chunk * 8192 +
                                                        sw128_offset(t, byte0 + v * 16));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          x[v * 8 + 2 * u] = __low2float(p2[u]);
          x[v * 8 + 2 * u + 1] = __high2float(p2[u]);
        }
      }
      constexpr float LOG2E = 1.4426950408889634f;
      auto ex2 = [](float v) {
        float y;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(v));
        return y;
      };
      float inv;
      if (a.phi == 1) {  // elu(x) + 1
#pragma unroll
        for (int e = 0; e < NE; ++e) x[e] = x[e] > 0.f ? x[e] + 1.f : ex2(x[e] * LOG2E);
        inv = (t < cnt) ? 1.f : 0.f;
      } else {           // softmax over d
        float m = x[0];
#pragma unroll
        for (int e = 1; e < NE; ++e) m = fmaxf(m, x[e]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          x[e] = ex2((x[e] - m) * LOG2E);
          sum += x[e];
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        inv = (t < cnt) ? 1.f / sum : 0.f;
      }
      // padding tokens of a partial block get phi = 0 (inv = 0)
#pragma unroll
      for (int v = 0; v < NE / 8; ++v) {
        uint4 q;
        q.x = pack_bf16x2(x[v * 8 + 0] * inv, x[v * 8 + 1] * inv);
        q.y = pack_bf16x2(x[v * 8 + 2] * inv, x[v * 8 + 3] * inv);
        q.z = pack_bf16x2(x[v * 8 + 4] * inv, x[v * 8 + 5] * inv);
        q.w = pack_bf16x2(x[v * 8 + 6] * inv, x[v * 8 + 7] * inv);
        *reinterpret_cast<uint4*>(sK + chunk * 8192 + sw128_offset(t, byte0 + v * 16)) = q;
      }
    }
    if (proj) {  // V'^T = D1 (row o = output feature, 64 token columns) in place of V
      const bool ok = mbar_wait(mma_bar, mma_phase & 1, a.err, DEV_TIMEOUT_MMA);
      ++mma_phase;
      if (!__syncthreads_and(ok)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tD1 + lane_off, r0);
      tmem_ld32(tD1 + lane_off + 32, r1);
      tmem_ld_wait();
      if (my_row >= 0) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 q;
          q.x = pack_bf16x2(__uint_as_float(r0[8 * v + 0]), __uint_as_float(r0[8 * v + 1]));
          q.y = pack_bf16x2(__uint_as_float(r0[8 * v + 2]), __uint_as_float(r0[8 * v + 3]));
          q.z = pack_bf16x2(__uint_as_float(r0[8 * v + 4]), __uint_as_float(r0[8 * v + 5]));
          q.w = pack_bf16x2(__uint_as_float(r0[8 * v + 6]), __uint_as_float(r0[8 * v + 7]));
          *reinterpret_cast<uint4*>(sV + sw128_offset(my_row, v * 16)) = q;
          q.x = pack_bf16x2(__uint_as_float(r1[8 * v + 0]), __uint_as_float(r1[8 * v + 1]));
          q.y = pack_bf16x2(__uint_as_float(r1[8 * v + 2]), __uint_as_float(r1[8 * v + 3]));
          q.z = pack_bf16x2(__uint_as_float(r1[8 * v + 4]), __uint_as_float(r1[8 * v + 5]));
          q.w = pack_bf16x2(__uint_as_float(r1[8 * v + 6]), __uint_as_float(r1[8 * v + 7]));
          *reinterpret_cast<uint4*>(sV + sw128_offset(my_row, 64 + v * 16)) = q;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(D, D, !proj, true);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = proj ? sdesc_sw128(smem_u32(sV) + k * 32, 16, 1024)
                                 : sdesc_sw128(smem_u32(sV) + k * 2048, 8192, 1024);
        const uint64_t bd = sdesc_sw128(smem_u32(sK) + k * 2048, 8192, 1024);
        umma_ss(tD2, ad, bd, id, k > 0);
      }
      umma_commit(mma_bar);
      // the block two ahead into the stage that the previous block used, once
      // that block's store has finished reading it
      const int nx = item + 2 * (int)gridDim.x;
      if (nx < a.nitems) {
        bulk_wait_read_all();
        issue_load(nx, (n + 2) % L::NST);
        ++n_issued;
      }
    }
    // z_j = column sums of phi(K_j) (the bf16 values the MMA consumes): eight
    // partial sums, so that the 64 shared-memory loads are not one dependent chain
    float z = 0.f;
    if (tid < D) {
      const int chunk = tid / 64, byte = (tid % 64) * 2;
      float zp[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) zp[q] = 0.f;
#pragma unroll
      for (int t = 0; t < 64; ++t)
        zp[t & 7] += __bfloat162float(
            *reinterpret_cast<const __nv_bfloat16*>(sK + chunk * 8192 + sw128_offset(t, byte)));
      z = ((zp[0] + zp[1]) + (zp[2] + zp[3])) + ((zp[4] + zp[5]) + (zp[6] + zp[7]));
    }
    {
      const bool ok = mbar_wait(mma_bar, mma_phase & 1, a.err, DEV_TIMEOUT_MMA);
      ++mma_phase;
      if (!__syncthreads_and(ok)) break;
    }
    tc_fence_after();
    // (h_j W^T)^T rows -> the stage as [chunk of a][row b][128 B] (swizzled)
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tD2 + lane_off + c0, r);
      tmem_ld_wait();
      if (my_row >= 0) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 q;
          q.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
          q.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
          q.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
          q.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
          const int col = c0 + 8 * v;  // a index of this 16-byte group
          *reinterpret_cast<uint4*>(sK + (col / 64) * (D * 128) +
                                    sw128_offset(my_row, (col % 64) * 2)) = q;
        }
      }
    }
    __nv_bfloat16* zout = a.hz + ((int64_t)bh * a.Tkv + j) * (int64_t)(D * D + D) + D * D;
    if (tid < D) zout[tid] = __float2bfloat16(z);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
#pragma unroll
      for (int c = 0; c < L::CH; ++c) tma_store_4d(&mapO, sK + c * (D * 128), c * 64, 0, j, bh);
      bulk_commit_group();
    }
  }
  if (tid == 0) {
    // loads still in flight after an early exit land before the CTA leaves
    for (int k = n; k < n_issued; ++k)
      if (!mbar_wait(&tma_bar[k % L::NST], (k / L::NST) & 1, a.err, DEV_TIMEOUT_TMA)) break;
    bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

template <int D>
static cudaError_t launch_kv_prep_t(const CUtensorMap& mapK, const CUtensorMap& mapV,
                                    const CUtensorMap& mapO, const KvPrepArgs& a, cudaStream_t s,
                                    int ctas_per_sm) {
  using L = KvSmem<D>;
  cudaError_t e = cudaFuncSetAttribute(kv_prep_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = min(a.nitems, (ctas_per_sm == 1 ? 1 : 2) * sms);
  kv_prep_kernel<D><<<grid, 128, L::ALLOC, s>>>(mapK, mapV, mapO, a);
  return cudaGetLastError();
}

cudaError_t launch_kv_prep(const CUtensorMap& mapK, const CUtensorMap& mapV, const CUtensorMap& mapO,
                           const KvPrepArgs& a, int D, cudaStream_t s, int ctas_per_sm) {
  return D == 128 ? launch_kv_prep_t<128>(mapK, mapV, mapO, a, s, ctas_per_sm)
                  : launch_kv_prep_t<64>(mapK, mapV, mapO, a, s, ctas_per_sm);
}

}  // namespace sla
