// Marginal aggregation ("SLA: Beyond Sparsity in Diffusion Transformers via
// Fine-Tunable Sparse-Linear Attention", §2 Q2 step 3 and Fig. 4: for every
// marginal block, H_i += h_j and Z_i += z_j).
//
// Summing the marginal h_j row by row would read n_m * d^2 values per query
// block.  Instead all rows are formed at once as one dense product per head,
//     [H_i^T | Z_i] = sum_j Mmarg[i][j] [h_j^T | z_j],   Mmarg = (M_c == 0),
// a (T_q x T_kv) x (T_kv x (d^2 + d)) GEMM on the tensor cores (0/1 weights
// are exact in bf16, accumulation in fp32).
//
//   marg_matrix_kernel  M_c (int8) -> Mmarg (bf16 0/1, rows padded to T_kvp); all
//                       ones for the variant whose linear branch covers every block
//   marg_gemm_kernel    persistent, 128 x 256 output tiles, K step 64,
//                       4-stage TMA ring, two TMEM accumulators; warp 0 loads,
//                       warp 1 issues tcgen05.mma, warps 2-5 drain TMEM into a
//                       swizzled bf16 staging tile (128 columns at a time)
//                       that one thread stores with TMA (whole 128-byte
//                       lines), while the next tile accumulates.
#include "kernels.cuh"

namespace sla {

__global__ void marg_matrix_kernel(const int8_t* __restrict__ mc, __nv_bfloat16* __restrict__ mm,
                                   int BH, int Tq, int Tkv, int Tkvp, bool all) {
  const int64_t total = (int64_t)BH * Tq * Tkvp;
  const __nv_bfloat16 one = __float2bfloat16(1.f), zero = __float2bfloat16(0.f);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(e % Tkvp);
    const int64_t row = e / Tkvp;  // bh * Tq + i
    mm[e] = (j < Tkv && (all || mc[row * Tkv + j] == 0)) ? one : zero;
  }
}

// The transpose for the backward: MmargT[bh][j][i] = Mmarg[bh][i][j], rows
// padded to T_qp (the dh_j = sum_i dH_i product of the linear backward).
__global__ void marg_matrix_t_kernel(const int8_t* __restrict__ mc, __nv_bfloat16* __restrict__ mt,
                                     int BH, int Tq, int Tkv, int Tqp, bool all) {
  const int64_t total = (int64_t)BH * Tkv * Tqp;
  const __nv_bfloat16 one = __float2bfloat16(1.f), zero = __float2bfloat16(0.f);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % Tqp);
    const int64_t r = e / Tqp;  // bh * Tkv + j
    const int j = (int)(r % Tkv);
    const int64_t bh = r / Tkv;
    mt[e] = (i < Tq && (all || mc[(bh * Tq + i) * Tkv + j] == 0)) ? one : zero;
  }
}

namespace {
// Four 48 KB stages (192 KB of loads in flight per SM: the [h|z] tiles come
// partly from HBM, and fewer bytes in flight left the tensor pipe waiting) and
// a 32 KB staging tile that takes the 256 output columns in two halves.
constexpr int BM = 128, BN = 256, BK = 64, NST = 4;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BK * BN * 2;   // 32 KB
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int OFF_OUT = NST * STAGE;   // bf16 staging: 2 chunks of [128 rows][64 columns]
constexpr int OUT_BYTES = BM * 128 * 2;
constexpr int OFF_BAR = OFF_OUT + OUT_BYTES;
constexpr int SMEM = OFF_BAR + 256 + 1024;

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
}  // namespace

// Persistent: CTA c takes tiles c, c + G, c + 2G, ... with the M tile index
// fastest, so CTAs running at the same time share their B (h) tiles in L2.
// Two TMEM accumulators (2 x 256 columns): the epilogue of one tile overlaps
// the main loop of the next.
__global__ void __launch_bounds__(192, 1) marg_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                                                           const __grid_constant__ CUtensorMap mapB,
                                                           const __grid_constant__ CUtensorMap mapO,
                                                           MargArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* acc_full = empty + NST;   // [2]
  uint64_t* acc_empty = acc_full + 2; // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int Mt = (a.Tq + BM - 1) / BM, Nt = (a.NN + BN - 1) / BN;
  const int ntiles = Mt * Nt * a.BH;

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], 128);
    }
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = *tslot;

  if (w == 0) {
    if (ln == 0) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m0 = (t % Mt) * BM, n0 = ((t / Mt) % Nt) * BN, bh = t / (Mt * Nt);
        const int nvalid_chunks = min(4, (a.NN - n0 + 63) / 64);
        for (int kt = 0; kt < a.ktiles; ++kt, ++it) {
          const int s = it % NST;
          if (it >= NST && !mbar_wait(&empty[s], ((it / NST) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
            ok = false;
            break;
          }
          uint8_t* sA = sm + s * STAGE;
          uint8_t* sB = sA + A_BYTES;
          mbar_arrive_expect_tx(&full[s], A_BYTES + nvalid_chunks * 8192);
          tma_load_3d(sA, &mapA, &full[s], kt * BK, m0, bh);
          for (int c = 0; c < nvalid_chunks; ++c)
            tma_load_3d(sB + c * 8192, &mapB, &full[s], n0 + c * 64, kt * BK, bh);
        }
      }
    }
  } else if (w == 1) {
    if (ln == 0) {
      const uint32_t id = idesc_bf16(BM, BN, false, true);
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        if (lt >= 2 && !mbar_wait(&acc_empty[ab], ((lt >> 1) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tacc + 256 * ab;
        for (int kt = 0; kt < a.ktiles; ++kt, ++it) {
          const int s = it % NST;
          if (!mbar_wait(&full[s], (it / NST) & 1, a.err, DEV_TIMEOUT_TMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(sm + s * STAGE);
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(sA + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sB + k * 2048, 8192, 1024);
            umma_ss(d, ad, bd, id, (kt > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[ab]);
      }
    }
  } else {
    const int q4 = w & 3;
    const int row = 32 * q4 + ln;
    const bool leader = tid == 64;  // issues the TMA stores of the output tile
    uint8_t* sO = sm + OFF_OUT;
    // Every epilogue warp runs every tile's two named barriers, also after a
    // wait gave up (then it only skips the work), so none is left waiting.
    bool ok = true;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int m0 = (t % Mt) * BM, n0 = ((t / Mt) % Nt) * BN, bh = t / (Mt * Nt);
      const int ab = lt & 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (lt >> 1) & 1, a.err, DEV_TIMEOUT_MMA));
      tc_fence_after();
      const uint32_t taddr = tacc + 256 * ab + ((uint32_t)(32 * q4) << 16);
      for (int hf = 0; hf < 2; ++hf) {
        // the previous TMA stores have finished reading the staging tile
        if (leader) bulk_wait_read_all();
        epi_sync();
        if (ok) {
#pragma unroll 1
          for (int c0 = 128 * hf; c0 < 128 * hf + 128; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c0, r);
            tmem_ld_wait();
            // row `row` of staging chunk (c0 / 64) % 2, 16-byte units (c0 % 64) / 8 .. + 3, 128-byte swizzle
            uint8_t* chunk = sO + ((c0 >> 6) & 1) * (BM * 128) + row * 128;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int unit = ((c0 & 63) >> 3) + v;
              uint4 q;
              q.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              q.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              q.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              q.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              *reinterpret_cast<uint4*>(chunk + ((unit ^ (row & 7)) << 4)) = q;
            }
          }
          if (hf == 1) {
            // the accumulator has been read: the MMA warp may reuse it
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
          }
          fence_proxy_async_smem();
        }
        epi_sync();
        if (leader && ok) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col = n0 + 128 * hf + 64 * c;
            if (col < a.NN) tma_store_3d(&mapO, sO + c * (BM * 128), col, m0, bh);
          }
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tacc, 512);
  }
}

// ---------------------------------------------------------------------------
// The same product for T_kv <= 512 with the 0/1 operand in TMEM.
//
// With both operands in shared memory every MMA re-reads the 0/1 tile, and
// shared memory (128 B per clock per SM) carries the TMA writes, the MMA reads
// and the epilogue staging: about 1.75x what the tensor pipe needs.  Here a CTA
// owns one (head, 128 query blocks) row band at a time: its 0/1 rows
// Mmarg[i][0 .. T_kv) sit in TMEM columns [0, 256) as bf16 pairs, built by
// the epilogue warps straight from M_c (no 0/1 matrix in memory), and the CTA
// walks a contiguous range of 128-column output tiles of that band, so only
// the [h|z] rows stream through shared memory (read once by the MMA).  CTAs
// come in groups of ceil(T_q / 128), one per band of the same head, that walk
// the same column tiles in step: each [h|z] tile is read from HBM once and
// from L2 by the group's other CTAs.
// Accumulators: two 128-column TMEM buffers at [256, 512); the epilogue of one
// tile overlaps the main loop of the next, through two staging tiles stored
// with TMA.  One CTA per SM.
// ---------------------------------------------------------------------------
namespace {
constexpr int TM_BN = 128, TM_BK = 64, TM_NST = 10;  // 160 KB of [h|z] loads in flight
constexpr int TM_STAGE = TM_BK * TM_BN * 2;        // 16 KB: [2 chunks][64 K rows][128 B]
constexpr int TM_OFF_OUT = TM_NST * TM_STAGE;      // staging: 2 x [2 chunks][128 rows][128 B]
constexpr int TM_OUT = 128 * TM_BN * 2;            // 32 KB
constexpr int TM_OFF_BAR = TM_OFF_OUT + 2 * TM_OUT;
constexpr int TM_SMEM = TM_OFF_BAR + 256 + 1024;
constexpr uint32_t TM_COL_ACC = 256;
}  // namespace

__global__ void __launch_bounds__(192, 1) marg_gemm_tm_kernel(const __grid_constant__ CUtensorMap mapB,
                                                              const __grid_constant__ CUtensorMap mapO,
                                                              MargArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + TM_OFF_BAR);
  uint64_t* empty = full + TM_NST;
  uint64_t* acc_full = empty + TM_NST;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* a_full = acc_empty + 2;     // the band's 0/1 rows are in TMEM
  uint32_t* tslot = reinterpret_cast<uint32_t*>(a_full + 1);
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int Mt = (a.Tq + 127) / 128, Nt = (a.NN + TM_BN - 1) / TM_BN;
  // group g (of G) takes a contiguous range of the (head, column tile) pairs;
  // CTA mi of the group computes row band mi of each
  const int G = gridDim.x / Mt, g = blockIdx.x / Mt, mi = blockIdx.x % Mt;
  const int64_t W = (int64_t)a.BH * Nt;
  const int64_t j0 = W * g / G, j1 = W * (g + 1) / G;  // j = bh * Nt + column tile
  const int m0 = mi * 128;
  const int ktiles = a.ktiles;
  auto band = [&](int64_t j) { return j / Nt; };  // the head

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < TM_NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], 128);
    }
    mbar_init(a_full, 128);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (w == 0) {
    // ------------------------------------------------------------ TMA producer
    if (ln == 0) {
      tma_prefetch_desc(&mapB);
      int it = 0;
      bool ok = true;
      for (int64_t j = j0; j < j1 && ok; ++j) {
        const int n0 = (int)(j % Nt) * TM_BN, bh = (int)(j / Nt);
        const int nvalid = min(2, (a.NN - n0 + 63) / 64);
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % TM_NST;
          if (it >= TM_NST && !mbar_wait(&empty[s], ((it / TM_NST) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
            ok = false;
            break;
          }
          uint8_t* sB = sm + s * TM_STAGE;
          mbar_arrive_expect_tx(&full[s], nvalid * 8192);
          for (int c = 0; c < nvalid; ++c)
            tma_load_3d(sB + c * 8192, &mapB, &full[s], n0 + c * 64, kt * TM_BK, bh);
        }
      }
    }
  } else if (w == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (ln == 0) {
      const uint32_t id = idesc_bf16(128, TM_BN, false, true);
      int it = 0, lt = 0, la = 0;
      bool ok = true;
      for (int64_t j = j0; j < j1 && ok; ++j, ++lt) {
        if (j == j0 || band(j) != band(j - 1)) {
          if (!mbar_wait(a_full, la & 1, a.err, DEV_TIMEOUT_SYNC)) break;
          ++la;
        }
        const int ab = lt & 1;
        if (lt >= 2 && !mbar_wait(&acc_empty[ab], ((lt >> 1) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        tc_fence_after();
        const uint32_t d = tbase + TM_COL_ACC + TM_BN * ab;
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % TM_NST;
          if (!mbar_wait(&full[s], (it / TM_NST) & 1, a.err, DEV_TIMEOUT_TMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sB = smem_u32(sm + s * TM_STAGE);
#pragma unroll
          for (int kk = 0; kk < TM_BK / 16; ++kk)
            umma_ts(d, tbase + kt * 32 + kk * 8, sdesc_sw128(sB + kk * 2048, 8192, 1024), id,
                    (kt > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[ab]);
      }
    }
  } else {
    // ------------------------------------------------------------ 0/1 rows and epilogue
    const int q4 = w & 3;
    const int row = 32 * q4 + ln;
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const bool leader = tid == 64;  // issues the TMA stores
    // 16-byte loads of M_c rows when every row starts on a 16-byte boundary
    const bool fast = (a.Tkv % 16) == 0 && (reinterpret_cast<uintptr_t>(a.mc) & 15u) == 0;
    // Every epilogue warp runs every tile's named barriers, also after a wait
    // gave up (then it only skips the work), so none is left waiting.
    bool ok = true;
    const int64_t cnt = j1 - j0;
    for (int64_t t = 0; t <= cnt; ++t) {
      bool waited = false;
      if (t < cnt && (t == 0 || band(j0 + t) != band(j0 + t - 1))) {
        // the previous tile's MMAs (the last readers of the old rows) are complete
        if (t > 0 && ok) {
          ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[(t - 1) & 1], ((t - 1) >> 1) & 1, a.err,
                                                 DEV_TIMEOUT_MMA));
          waited = true;
        }
        tc_fence_after();
        if (ok) {
          const int bh = (int)band(j0 + t), i = m0 + row;
          const bool live = i < a.Tq;
          const int8_t* src = a.mc + ((int64_t)bh * a.Tq + (live ? i : 0)) * a.Tkv;
          // columns [32 c0, 32 c0 + 32) hold K = 64 c0 .. 64 c0 + 63 as bf16 pairs
          for (int c0 = 0; c0 < ktiles; ++c0) {
            uint32_t v[32];
            const int k0 = 64 * c0;
            if (fast && live && k0 + 64 <= a.Tkv) {
              const uint4* p = reinterpret_cast<const uint4*>(src + k0);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 b = __ldg(p + q);
                const uint32_t wd[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const uint32_t b0 = (wd[e] >> (16 * h)) & 0xffu, b1 = (wd[e] >> (16 * h + 8)) & 0xffu;
                    v[8 * q + 2 * e + h] = ((a.all || b0 == 0) ? 0x3F80u : 0u) |
                                           ((a.all || b1 == 0) ? 0x3F800000u : 0u);
                  }
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int k = k0 + 2 * c;
                const bool m0 = live && k < a.Tkv && (a.all || src[k] == 0);
                const bool m1 = live && k + 1 < a.Tkv && (a.all || src[k + 1] == 0);
                v[c] = (m0 ? 0x3F80u : 0u) | (m1 ? 0x3F800000u : 0u);
              }
            }
            tmem_st32(tbase + lane_off + 32 * c0, v);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(a_full);
      }
      if (t == 0) continue;
      // ---- epilogue of tile t - 1
      const int64_t jj = j0 + t - 1;
      const int pl = (int)(t - 1);
      const int n0 = (int)(jj % Nt) * TM_BN, bh = (int)(jj / Nt);
      const int ab = pl & 1;
      if (ok && !waited)
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (pl >> 1) & 1, a.err, DEV_TIMEOUT_MMA));
      tc_fence_after();
      uint8_t* sO = sm + TM_OFF_OUT + ab * TM_OUT;
      // the store issued two tiles ago from this staging tile has read it
      if (leader) bulk_wait_read_1();
      epi_sync();
      if (ok) {
        const uint32_t taddr = tbase + TM_COL_ACC + TM_BN * ab + lane_off;
#pragma unroll 1
        for (int c0 = 0; c0 < TM_BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(taddr + c0, r);
          tmem_ld_wait();
          uint8_t* chunk = sO + (c0 >> 6) * (128 * 128) + row * 128;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int unit = ((c0 & 63) >> 3) + v;
            uint4 q;
            q.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
            q.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            q.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            q.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            *reinterpret_cast<uint4*>(chunk + ((unit ^ (row & 7)) << 4)) = q;
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[ab]);
        fence_proxy_async_smem();
      }
      epi_sync();
      if (leader && ok) {
#pragma unroll
        for (int c = 0; c < TM_BN / 64; ++c)
          if (n0 + 64 * c < a.NN) tma_store_3d(&mapO, sO + c * (128 * 128), n0 + 64 * c, m0, bh);
        bulk_commit_group();
      }
    }
    if (leader) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

cudaError_t launch_marg_matrix(const int8_t* mc, __nv_bfloat16* mm, int BH, int Tq, int Tkv,
                               int Tkvp, bool all, cudaStream_t s) {
  const int64_t total = (int64_t)BH * Tq * Tkvp;
  const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
  marg_matrix_kernel<<<blocks, 256, 0, s>>>(mc, mm, BH, Tq, Tkv, Tkvp, all);
  return cudaGetLastError();
}

cudaError_t launch_marg_matrix_t(const int8_t* mc, __nv_bfloat16* mt, int BH, int Tq, int Tkv,
                                 int Tqp, bool all, cudaStream_t s) {
  const int64_t total = (int64_t)BH * Tkv * Tqp;
  const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
  marg_matrix_t_kernel<<<blocks, 256, 0, s>>>(mc, mt, BH, Tq, Tkv, Tqp, all);
  return cudaGetLastError();
}

cudaError_t launch_marg_gemm(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapO,
                             const MargArgs& a, int BH, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(marg_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = ((a.NN + BN - 1) / BN) * ((a.Tq + BM - 1) / BM) * BH;
  MargArgs b = a;
  b.BH = BH;
  marg_gemm_kernel<<<ntiles < sms ? ntiles : sms, 192, SMEM, s>>>(mapA, mapB, mapO, b);
  return cudaGetLastError();
}

cudaError_t launch_marg_gemm_tm(const CUtensorMap& mapB, const CUtensorMap& mapO, const MargArgs& a, int BH,
                                cudaStream_t s) {
  if (a.Tkv > kMargTmemMaxTkv || a.ktiles * 64 < a.Tkv) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(marg_gemm_tm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TM_SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // groups of Mt CTAs (one per row band), as many groups as fit the SMs, at
  // most one per (head, column tile)
  const int Mt = (a.Tq + 127) / 128;
  const int64_t W = (int64_t)((a.NN + TM_BN - 1) / TM_BN) * BH;
  int64_t G = sms / Mt;
  if (G < 1) G = 1;
  if (G > W) G = W;
  MargArgs b = a;
  b.BH = BH;
  marg_gemm_tm_kernel<<<(int)(G * Mt), 192, TM_SMEM, s>>>(mapB, mapO, b);
  return cudaGetLastError();
}

}  // namespace sla
