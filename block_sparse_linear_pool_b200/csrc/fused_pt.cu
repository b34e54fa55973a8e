// Persistent fused SLA / SLA2 forward ("SLA: Beyond Sparsity in Diffusion
// Transformers via Fine-Tunable Sparse-Linear Attention", §2 Q2 steps 3-4 and
// Fig. 4 "Fused kernel"; "SLA2: Sparse-Linear Attention with Learnable Routing
// and QAT", §3), bf16 Q K^T and P V.
//
// A tile is 128 query rows = two query blocks of one head (chosen by the
// pairing kernels for overlapping critical lists), so every tcgen05.mma runs at
// M = 128.  The tile walks the union of its two blocks' critical lists
// (precomputed per tile by tile_union_kernel, below), one key block per entry:
// S_k = Q K_j^T into one of two TMEM score buffers, the softmax writes P_k over
// S_k, O += P_k V_j.  A key block that is critical for only one of the two query
// blocks is masked out of the other half (probability 0).  K and V tiles stream
// through two-slot rings, K one entry ahead of V.
//
// The linear branch is folded into the same accumulator: after the last P V the
// softmax threads write P' = phi~(q) * (w_l / w_s) into the score columns and the
// MMA warp adds P'_a H_a^T + P'_b H_b^T to O (one MMA chain per query block, the
// other half's rows zero), so that the epilogue's O w_s is
//     w_s O^s_acc + w_l phi~(q) H_i      (w_s = 1/l, w_l = 1/den for SLA;
//                                        w_s = a/l, w_l = (1-a)/den for SLA2)
// with phi~(q) H / (phi~(q) Z + s eps) = phi(q) H / (phi(q) Z + eps) exactly.
//
// CTAs are persistent (two per SM: 256 TMEM columns and ~100 KB of shared memory
// each) and take tiles blockIdx.x, blockIdx.x + gridDim.x, ...: the next tile's
// union record, Q tile and first K tiles load while the current tile finishes,
// and its H tiles and the next tile's Q are prefetched into L2 early.
//
//   warp 0      TMA producer: the tile's union record (bulk copy, two buffers),
//               Q tile + Z rows, K and V of each entry, then H_a^T through the K
//               ring and H_b^T through the V ring (one 64-column chunk per slot)
//   warp 1      MMA issuer (one thread; the shared-memory descriptors are
//               formed once and advanced by constants): S, P V, and the two
//               linear-branch chains.  S_{k+1} is issued as soon as P_{k-1} V
//               is, so that it runs beside the softmax of entry k: the two
//               score buffers are what keeps the tensor pipe fed within a CTA.
//   warps 2-5   one query row per thread: online softmax with exp2 (lazy
//               rescale of O only when the running max grows by more than 2^8;
//               the scaling and the row sum in paired fp32 instructions, the
//               row maximum with three-input max), P over S in TMEM; then
//               (training forward) the row's LSE and its sparse-branch output
//               o^s from O before the linear term joins it, phi~(q), P', and
//               the epilogue
//
// TMEM: S_0 in columns [0, 64), S_1 in [64, 128) (P', after the loop, over
// [0, d)), O in [128, 128 + d).
#include "kernels.cuh"

namespace sla {

namespace {

constexpr uint32_t PT_COL_S = 0, PT_COL_O = 128;
constexpr float PT_RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr float PT_LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float pt_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct PtSmem {
  static constexpr int CH = D / 64;              // 64-column chunks of d
  static constexpr int Q_BYTES = 128 * D * 2;    // [chunk][128 rows][128 B]
  static constexpr int KT_BYTES = 64 * D * 2;    // one ring slot: a key block of K or V,
                                                 // or one 64-column chunk of an H tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * KT_BYTES;
  static constexpr int OFF_Z = OFF_V + 2 * KT_BYTES;  // Z_a, Z_b: 2 x D bf16
  static constexpr int OFF_BAR = OFF_Z + 4 * D;
  static constexpr int OFF_U = OFF_BAR + 256;     // two union records
  static size_t bytes(int urec_bytes) { return (size_t)OFF_U + 2 * (size_t)urec_bytes + 1024; }
};
static_assert(64 * 128 * 2 == 128 * 128, "an H chunk ([d rows][64 columns]) fills one ring slot");

}  // namespace

// ---------------------------------------------------------------------------
// Per tile: the union of its two query blocks' critical lists, ascending, each
// entry j | flag << 14 (flag bit 0: critical for the first block, bit 1: for
// the second).  Record = uint16 [urec]: rec[0] = count, entries from rec[8].
// One warp per tile: the two lists as bitsets over the key blocks in shared
// memory, then a warp scan over the words writes the entries in order.
// ---------------------------------------------------------------------------
constexpr int UNION_WARPS = 4;
constexpr int UNION_MAX_WORDS = 128;  // T_kv <= 4096

__global__ void __launch_bounds__(32 * UNION_WARPS)
    tile_union_kernel(const int32_t* __restrict__ lut, const int2* __restrict__ pairs, int Tq, int Tkv, int nh,
                      int ntiles, int urec, uint16_t* __restrict__ out, int* __restrict__ err) {
  __shared__ uint32_t bits[UNION_WARPS][2][UNION_MAX_WORDS];
  const int wl = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const int t = blockIdx.x * UNION_WARPS + wl;
  if (t >= ntiles) return;
  const int W = (Tkv + 31) >> 5;
  uint32_t* ba = bits[wl][0];
  uint32_t* bb = bits[wl][1];
  for (int x = ln; x < W; x += 32) ba[x] = bb[x] = 0u;
  __syncwarp();
  const int npair = (Tq + 1) / 2;
  const int bh = t / npair;
  const int2 pr = pairs[t];
  const int32_t* la = lut + ((int64_t)bh * Tq + pr.x) * nh;
  const int32_t* lb = lut + ((int64_t)bh * Tq + (pr.y >= 0 ? pr.y : pr.x)) * nh;
  const int tot = pr.y >= 0 ? 2 * nh : nh;
  for (int e = ln; e < tot; e += 32) {
    const bool second = e >= nh;
    const int j = __ldg(second ? lb + (e - nh) : la + e);
    if (j < 0 || j >= Tkv) {
      atomicCAS(err, 0, DEV_BAD_INDEX);
      continue;
    }
    atomicOr(&(second ? bb : ba)[j >> 5], 1u << (j & 31));
  }
  __syncwarp();
  uint16_t* rec = out + (int64_t)t * urec;
  const int cap = urec - 8;
  int base = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int x = w0 + ln;
    const uint32_t wa = x < W ? ba[x] : 0u, wb = x < W ? bb[x] : 0u;
    uint32_t wu = wa | wb;
    const int cnt = __popc(wu);
    int pre = cnt;  // inclusive scan over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, pre, o);
      if (ln >= o) pre += y;
    }
    int pos = base + pre - cnt;
    while (wu) {
      const int bit = __ffs(wu) - 1;
      wu &= wu - 1;
      const uint32_t flag = ((wa >> bit) & 1u) | (((wb >> bit) & 1u) << 1);
      if (pos < cap) rec[8 + pos] = (uint16_t)((32 * x + bit) | (flag << 14));
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, pre, 31);
  }
  if (ln == 0) {
    if (base > cap) atomicCAS(err, 0, DEV_BAD_INDEX);
    rec[0] = (uint16_t)(base < cap ? base : cap);
  }
}

cudaError_t launch_tile_union(const int32_t* lut, const int2* pairs, int BH, int Tq, int Tkv, int nh, int urec,
                              uint16_t* out, int* err, cudaStream_t s) {
  const int ntiles = BH * ((Tq + 1) / 2);
  if (Tkv > 32 * UNION_MAX_WORDS) return cudaErrorInvalidValue;
  tile_union_kernel<<<(ntiles + UNION_WARPS - 1) / UNION_WARPS, 32 * UNION_WARPS, 0, s>>>(lut, pairs, Tq, Tkv, nh,
                                                                                      ntiles, urec, out, err);
  return cudaGetLastError();
}


// One softmax entry of one query row: the 64 scores of one critical key block
// in TMEM score buffer tS, the row's running max m (log2 units) and sum l.
// Writes P (bf16 pairs, keys 2c and 2c + 1 in column c) over the first 32
// columns of the buffer, then rescales O if the max grew by more than the
// threshold (after the scores have left the registers; O must first hold the
// previous entry's P V).  Returns false if a wait gave up.
template <int D>
__device__ __forceinline__ bool pt_softmax_entry(uint32_t tS, uint32_t tO, int nvalid, float sl2, float& m,
                                                 float& l, uint64_t* pv_prev, uint32_t pv_parity, int* err) {
  uint32_t pk[32];
  bool grow = false;
  float fsc = 1.f;
  {
    uint32_t s0[32], s1[32];
    tmem_ld32(tS, s0);
    tmem_ld32(tS + 32, s1);
    tmem_ld_wait();
    if (nvalid < 64) {  // partial last key block: its padding columns get -inf
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (c >= nvalid) s0[c] = __float_as_uint(-INFINITY);
        if (c + 32 >= nvalid) s1[c] = __float_as_uint(-INFINITY);
      }
    }
    // row maximum with three-input max: 64 -> 22 -> 8 -> 3 -> 1
    float t[22];
#pragma unroll
    for (int i = 0; i < 21; ++i) {
      const int e = 3 * i;  // values 0..31 from s0, 32..63 from s1
      const float v0 = __uint_as_float(e < 32 ? s0[e] : s1[e - 32]);
      const float v1 = __uint_as_float(e + 1 < 32 ? s0[e + 1] : s1[e + 1 - 32]);
      const float v2 = __uint_as_float(e + 2 < 32 ? s0[e + 2] : s1[e + 2 - 32]);
      t[i] = fmax3(v0, v1, v2);
    }
    t[21] = __uint_as_float(s1[31]);
#pragma unroll
    for (int i = 0; i < 7; ++i) t[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
    t[7] = t[21];
    t[0] = fmax3(t[0], t[1], t[2]);
    t[1] = fmax3(t[3], t[4], t[5]);
    const float mx = fmax3(t[0], t[1], fmaxf(t[6], t[7])) * sl2;
    const bool first = (m == -INFINITY);
    grow = !first && (mx - m > PT_RESCALE_THRESHOLD);
    if (first) m = mx;  // O and l of this row are still exactly 0
    if (grow) {
      fsc = pt_ex2(m - mx);
      m = mx;
    }
    // p = 2^(s sl2 - m): the scaling in pairs (one instruction, two roundings
    // identical to fmaf), the sum in pairs
    const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
    uint64_t u2[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float x0, x1, x2, x3;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2, nm2), x0, x1);
      f2_unpack(f2_fma(f2_pack(__uint_as_float(s1[2 * c]), __uint_as_float(s1[2 * c + 1])), sc2, nm2), x2, x3);
      const float p0 = pt_ex2(x0), p1 = pt_ex2(x1), p2 = pt_ex2(x2), p3 = pt_ex2(x3);
      pk[c] = pack_bf16x2(p0, p1);
      pk[16 + c] = pack_bf16x2(p2, p3);
      u2[c] = f2_add(f2_pack(p0, p1), f2_pack(p2, p3));
    }
#pragma unroll
    for (int st = 8; st >= 1; st >>= 1)
#pragma unroll
      for (int c = 0; c < st; ++c) u2[c] = f2_add(u2[c], u2[c + st]);
    float ul, uh;
    f2_unpack(u2[0], ul, uh);
    l = l * fsc + (ul + uh);
  }
  tmem_st32(tS, pk);
  if (__any_sync(0xffffffffu, grow)) {
    // the next P V waits for this entry's p_ready, so O is not written meanwhile
    if (!__all_sync(0xffffffffu, mbar_wait(pv_prev, pv_parity, err, DEV_TIMEOUT_MMA))) return false;
    tc_fence_after();
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(tO + c0, o);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * fsc);
      tmem_st32(tO + c0, o);
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(192, 2)
    sla_fused_pt_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapH,
                        const __grid_constant__ CUtensorMap mapZ, FusedArgs a) {
  using L = PtSmem<D>;
  constexpr int CH = L::CH;
  constexpr int KT = L::KT_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sK = sm + L::OFF_K;
  uint8_t* sV = sm + L::OFF_V;
  uint8_t* sZ = sm + L::OFF_Z;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_free = bars + 1;
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2]
  uint64_t* p_ready = bars + 12;  // [2]
  uint64_t* pv_done = bars + 14;  // [2]
  uint64_t* lin_ready = bars + 16;
  uint64_t* o_full = bars + 17;
  uint64_t* o_free = bars + 18;
  uint64_t* u_full = bars + 19;   // [2]
  uint64_t* u_free = bars + 21;   // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 23);
  const int urec = a.urec;  // uint16 per union record
  uint16_t* sU = reinterpret_cast<uint16_t*>(sm + L::OFF_U);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int npair = (a.Tq + 1) / 2;
  const int ntiles = a.BH * npair;

  if (w == 1) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 4);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&k_full[x], 1);
      mbar_init(&k_empty[x], 1);
      mbar_init(&v_full[x], 1);
      mbar_init(&v_empty[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[x], 4);
      mbar_init(&pv_done[x], 1);
      mbar_init(&u_full[x], 1);
      mbar_init(&u_free[x], 5);
    }
    mbar_init(lin_ready, 4);
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (w == 0) {
    // ------------------------------------------------------------ TMA producer
    if (ln == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      tma_prefetch_desc(&mapH);
      tma_prefetch_desc(&mapZ);
      uint32_t kuse = 0, vuse = 0;  // ring fills so far (slot = fill % 2)
      bool ok = true;
      // next fill of a ring: wait for the slot's previous use, then arm its full barrier
      auto claim = [&](uint64_t* full, uint64_t* empty, uint32_t n, uint32_t bytes) -> bool {
        if (n >= 2 && !mbar_wait(&empty[n & 1], ((n >> 1) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        mbar_arrive_expect_tx(&full[n & 1], bytes);
        return true;
      };
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const int ub = it & 1;
        uint16_t* u = sU + ub * urec;
        if (it >= 2 && !mbar_wait(&u_free[ub], ((it >> 1) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        mbar_arrive_expect_tx(&u_full[ub], urec * 2);
        bulk_load(u, a.ulist + (int64_t)tile * urec, urec * 2, &u_full[ub]);
        const int bh = tile / npair, p = tile % npair;
        const int b = bh / a.H, h = bh % a.H;
        const int2 pr = a.pairs[(int64_t)bh * npair + p];
        const int ia = pr.x, ibl = pr.y >= 0 ? pr.y : pr.x;
        // into L2 early: this tile's H tiles and the next tile's Q rows
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          tma_prefetch_l2_4d(&mapH, c * 64, 0, ia, bh);
          tma_prefetch_l2_4d(&mapH, c * 64, 0, ibl, bh);
        }
        if (tile + (int)gridDim.x < ntiles) {
          const int t2 = tile + gridDim.x, bh2 = t2 / npair;
          const int2 p2 = a.pairs[(int64_t)bh2 * npair + t2 % npair];
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            tma_prefetch_l2_4d(&mapQ, c * 64, 64 * p2.x, bh2 % a.H, bh2 / a.H);
            if (p2.y >= 0) tma_prefetch_l2_4d(&mapQ, c * 64, 64 * p2.y, bh2 % a.H, bh2 / a.H);
          }
        }
        // Q tile and Z rows (the previous tile's phi~(q) has been read from sQ)
        if (it >= 1 && !mbar_wait(q_free, (it - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        mbar_arrive_expect_tx(q_full, L::Q_BYTES + 2 * D * 2);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          tma_load_4d(sQ + c * 16384, &mapQ, q_full, c * 64, 64 * ia, h, b);
          tma_load_4d(sQ + c * 16384 + 8192, &mapQ, q_full, c * 64, 64 * ibl, h, b);
          tma_load_3d(sZ + c * 128, &mapZ, q_full, D * D + c * 64, ia, bh);
          tma_load_3d(sZ + (CH + c) * 128, &mapZ, q_full, D * D + c * 64, ibl, bh);
        }
        if (!mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) break;
        const int U = u[0];
        // K_k one entry ahead of V_{k-1}
        for (int k = 0; k <= U && ok; ++k) {
          if (k < U) {
            const int j = u[8 + k] & 0x3fff;
            if (!claim(k_full, k_empty, kuse, KT)) { ok = false; break; }
#pragma unroll
            for (int c = 0; c < CH; ++c)
              tma_load_4d(sK + (kuse & 1) * KT + c * 8192, &mapK, &k_full[kuse & 1], c * 64, 64 * j, h, b);
            ++kuse;
          }
          if (k >= 1) {
            const int j = u[8 + k - 1] & 0x3fff;
            if (!claim(v_full, v_empty, vuse, KT)) { ok = false; break; }
#pragma unroll
            for (int c = 0; c < CH; ++c)
              tma_load_4d(sV + (vuse & 1) * KT + c * 8192, &mapV, &v_full[vuse & 1], c * 64, 64 * j, h, b);
            ++vuse;
          }
        }
        // H_a^T through the K ring, H_b^T through the V ring: one [d rows][64 a]
        // chunk per slot
        for (int c = 0; c < CH && ok; ++c) {
          if (!claim(k_full, k_empty, kuse, KT)) { ok = false; break; }
          tma_load_4d(sK + (kuse & 1) * KT, &mapH, &k_full[kuse & 1], c * 64, 0, ia, bh);
          ++kuse;
        }
        for (int c = 0; c < CH && ok; ++c) {
          if (!claim(v_full, v_empty, vuse, KT)) { ok = false; break; }
          tma_load_4d(sV + (vuse & 1) * KT, &mapH, &v_full[vuse & 1], c * 64, 0, ibl, bh);
          ++vuse;
        }
      }
    }
  } else if (w == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (ln == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      const uint32_t id_l = idesc_bf16(128, D, false, false);
      const uint32_t tS = tbase + PT_COL_S, tO = tbase + PT_COL_O;
      // Descriptors of ring slot 0 (and of Q); a byte offset o inside shared
      // memory adds o >> 4 to the start-address field, which cannot carry out.
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);    // K tile or H_a chunk (K-major)
      const uint64_t dVk = sdesc_sw128(smem_u32(sV), 16, 1024);   // H_b chunk (K-major)
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 8192, 1024);  // V tile (MN-major)
      constexpr uint64_t SLOT = KT >> 4;
      uint32_t kuse = 0, vuse = 0, g = 0;  // ring uses, entries so far
      bool ok = true;
      int it = 0;
      // O += P_e V: entry e (global index ge) of tile it
      auto issue_pv = [&](uint32_t ge, bool first_of_tile) -> bool {
        if (!mbar_wait(&p_ready[ge & 1], (ge >> 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        // the previous tile's epilogue must have read O before it is overwritten
        if (first_of_tile && it > 0 && !mbar_wait(o_free, (it - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        if (!mbar_wait(&v_full[vuse & 1], (vuse >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) return false;
        tc_fence_after();
        const uint64_t dv = dV + (vuse & 1) * SLOT;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tO, tS + 64 * (ge & 1) + 8 * kk, dv + kk * (2048 >> 4), id_pv, (!first_of_tile || kk > 0) ? 1u : 0u);
        umma_commit(&pv_done[ge & 1]);
        umma_commit(&v_empty[vuse & 1]);
        ++vuse;
        return true;
      };
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const int ub = it & 1;
        if (!mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) break;
        const int U = sU[ub * urec];
        if (!mbar_wait(q_full, it & 1, a.err, DEV_TIMEOUT_TMA)) break;
        for (int k = 0; k < U; ++k) {
          const uint32_t ge = g + k;
          if (!mbar_wait(&k_full[kuse & 1], (kuse >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
          // score buffer ge & 1 still holds P_{ge-2}, whose P V this thread issued
          // earlier: tcgen05.mma ops of one thread run in issue order
          tc_fence_after();
          const uint64_t dk = dK + (kuse & 1) * SLOT;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tS + 64 * (ge & 1), dQ + ((kk / 4) * 16384 + (kk % 4) * 32) / 16,
                    dk + ((kk / 4) * 8192 + (kk % 4) * 32) / 16, id_s, kk > 0 ? 1u : 0u);
          umma_commit(&s_full[ge & 1]);
          umma_commit(&k_empty[kuse & 1]);
          ++kuse;
          if (k >= 1 && !issue_pv(ge - 1, k == 1)) { ok = false; break; }
        }
        if (ok && U >= 1) ok = issue_pv(g + U - 1, U == 1);
        if (!ok) break;
        g += U;
        // linear branch: O += P'_a H_a^T (K ring) + P'_b H_b^T (V ring)
        if (!mbar_wait(lin_ready, it & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        for (int t = 0; t < 2 && ok; ++t) {
          uint64_t* full = t == 0 ? k_full : v_full;
          uint64_t* empty = t == 0 ? k_empty : v_empty;
          uint32_t& use = t == 0 ? kuse : vuse;
          const uint64_t dbase = t == 0 ? dK : dVk;
          for (int c = 0; c < CH; ++c) {
            if (!mbar_wait(&full[use & 1], (use >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
            tc_fence_after();
            const uint64_t dh = dbase + (use & 1) * SLOT;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ts(tO, tS + t * (D / 2) + 8 * (4 * c + kk), dh + kk * (32 >> 4), id_l, 1u);
            umma_commit(&empty[use & 1]);
            ++use;
          }
        }
        if (!ok) break;
        umma_commit(o_full);
        mbar_arrive(&u_free[ub]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int q4 = w & 3;
    const int r = 32 * q4 + ln;
    const int half = r >> 6;
    const uint32_t bit = 1u << half;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    const uint32_t tS = tl + PT_COL_S, tO = tl + PT_COL_O;
    const float sl2 = a.scale_log2;
    uint32_t g = 0;
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const int ub = it & 1;
      const uint16_t* u = sU + ub * urec;
      if (!__all_sync(0xffffffffu, mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA))) break;
      const int U = u[0];
      const int bh = tile / npair, p = tile % npair;
      const int2 pr = a.pairs[(int64_t)bh * npair + p];
      const bool has_b = pr.y >= 0;
      const int blk = half == 0 ? pr.x : (has_b ? pr.y : pr.x);
      const float alpha = a.combine == 1 ? a.alpha[bh] : 1.f;
      const bool sparse_on = alpha != 0.f;  // SLA2 with alpha = 0: only the linear branch
      float m = -INFINITY, l = 0.f;
      for (int k = 0; k < U; ++k) {
        const uint32_t ge = g + k;
        const uint32_t ts = tS + 64 * (ge & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[ge & 1], (ge >> 1) & 1, a.err, DEV_TIMEOUT_MMA))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t f = u[8 + k];
        if (sparse_on && ((f >> 14) & bit)) {  // warp-uniform
          if (!pt_softmax_entry<D>(ts, tO, a.N - 64 * (int)(f & 0x3fff), sl2, m, l, &pv_done[(ge - 1) & 1],
                                   ((ge - 1) >> 1) & 1, a.err)) {
            ok = false;
            break;
          }
        } else {
          tmem_st32_zero(ts);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (ln == 0) mbar_arrive(&p_ready[ge & 1]);
      }
      if (!ok) break;
      g += U;
      // ---------------- linear branch: P' = phi~(q_r) * (w_l / w_s) over the score columns
      // the last P V must have read its P first; Q and Z are in sQ / sZ
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, a.err, DEV_TIMEOUT_MMA));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(q_full, it & 1, a.err, DEV_TIMEOUT_TMA));
      if (!ok) break;
      tc_fence_after();
      const int n = 64 * blk + (r & 63);
      const bool store = (n < a.N) && (half == 0 || has_b);
      if (a.lse || a.os) {
        // for the backward: the sparse branch alone (O holds only P V so far) and the
        // log-sum-exp of the row's scaled critical scores, sum_t exp(s_t) = 2^m l
        const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
        if (a.lse && store) a.lse[(int64_t)bh * a.N + n] = (m + log2f(l)) * 0.6931471805599453f;
        if (a.os) {
#pragma unroll 1
          for (int c0o = 0; c0o < D; c0o += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + c0o, ov);
            tmem_ld_wait();
            if (store) {
              float4* od = reinterpret_cast<float4*>(a.os + ((int64_t)bh * a.N + n) * D + c0o);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                od[v] = make_float4(__uint_as_float(ov[4 * v]) * inv_l, __uint_as_float(ov[4 * v + 1]) * inv_l,
                                    __uint_as_float(ov[4 * v + 2]) * inv_l, __uint_as_float(ov[4 * v + 3]) * inv_l);
            }
          }
        }
      }
      // e = phi~(q) as bf16 pairs; the denominator's sums use the rounded values
      uint32_t pe[D / 2];
      float esum = 0.f, edotz = 0.f;
      {
        float mq = -INFINITY;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(sQ + (c / 8) * 16384 + sw128_offset(r, (c % 8) * 16));
          pe[4 * c] = v.x;
          pe[4 * c + 1] = v.y;
          pe[4 * c + 2] = v.z;
          pe[4 * c + 3] = v.w;
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) mq = fmaxf(mq, fmaxf(__low2float(p2[e]), __high2float(p2[e])));
        }
        // softmax over d: e = 2^((q - max q) log2 e), phi = e / sum(e);
        // elu + 1: e = phi itself, and the denominator's sum is 1
        const bool elu = a.phi == 1;
        const float nmq = -mq * PT_LOG2E;
        const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(sZ + (half == 1 ? CH * 128 : 0));
#pragma unroll
        for (int c = 0; c < D / 2; ++c) {
          const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
          const float x0 = __low2float(q2), x1 = __high2float(q2);
          const float e0 = elu ? (x0 > 0.f ? x0 + 1.f : pt_ex2(x0 * PT_LOG2E)) : pt_ex2(fmaf(x0, PT_LOG2E, nmq));
          const float e1 = elu ? (x1 > 0.f ? x1 + 1.f : pt_ex2(x1 * PT_LOG2E)) : pt_ex2(fmaf(x1, PT_LOG2E, nmq));
          pe[c] = pack_bf16x2(e0, e1);
          const __nv_bfloat162 eb = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
          const __nv_bfloat162 zb = z2[c];
          esum += __low2float(eb) + __high2float(eb);
          edotz = fmaf(__low2float(eb), __low2float(zb), fmaf(__high2float(eb), __high2float(zb), edotz));
        }
        if (elu) esum = 1.f;
      }
      // sQ and sZ have been read: the producer may load the next tile's Q
      __syncwarp();
      if (ln == 0) mbar_arrive(q_free);
      const float den = edotz + esum * a.eps;
      const float wl = (a.combine == 1 ? 1.f - alpha : 1.f) / den;
      const float ws = (l > 0.f) ? alpha / l : 0.f;  // alpha = 1 for SLA
      const float pscale = ws > 0.f ? wl / ws : wl;
      const float omul = ws > 0.f ? ws : 1.f;
#pragma unroll
      for (int c = 0; c < D / 2; ++c) {
        const __nv_bfloat162 eb = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
        pe[c] = pack_bf16x2(__low2float(eb) * pscale, __high2float(eb) * pscale);
      }
      // P'_a over columns [0, D/2), P'_b over [D/2, D): this row's half carries phi~(q)
#pragma unroll
      for (int c0p = 0; c0p < D / 2; c0p += 32) {
        uint32_t chunk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) chunk[c] = pe[c0p + c];
        tmem_st32(tS + half * (D / 2) + c0p, chunk);
        tmem_st32_zero(tS + (1 - half) * (D / 2) + c0p);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (ln == 0) mbar_arrive(lin_ready);
      // ---------------- epilogue: O w_s (+ bias)
      if (!__all_sync(0xffffffffu, mbar_wait(o_full, it & 1, a.err, DEV_TIMEOUT_MMA))) { ok = false; break; }
      tc_fence_after();
      {
        const int b = bh / a.H, h = bh % a.H;
        __nv_bfloat16* orow = a.O + (int64_t)b * a.so0 + (int64_t)h * a.so1 + (int64_t)n * a.so2;
#pragma unroll 1
        for (int c0o = 0; c0o < D; c0o += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + c0o, ov);
          tmem_ld_wait();
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0o);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int c = 8 * v + e;
                const float bias = (a.combine == 0 && a.proj_b) ? __ldg(a.proj_b + c0o + c) : 0.f;
                y[e] = __uint_as_float(ov[c]) * omul + bias;
              }
              dst[v] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                                  pack_bf16x2(y[6], y[7]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (ln == 0) {
        mbar_arrive(o_free);
        mbar_arrive(&u_free[ub]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

size_t fused_pt_smem_bytes(int D, int urec) {
  return D == 128 ? PtSmem<128>::bytes(urec * 2) : PtSmem<64>::bytes(urec * 2);
}

template <int D>
static cudaError_t launch_fused_pt_t(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                     const CUtensorMap& mapH, const CUtensorMap& mapZ, const FusedArgs& a,
                                     int nsm, cudaStream_t s) {
  const size_t smem = PtSmem<D>::bytes(a.urec * 2);
  cudaError_t e = cudaFuncSetAttribute(sla_fused_pt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntiles = a.BH * ((a.Tq + 1) / 2);
  const int grid = ntiles < 2 * nsm ? ntiles : 2 * nsm;
  sla_fused_pt_kernel<D><<<grid, 192, smem, s>>>(mapQ, mapK, mapV, mapH, mapZ, a);
  return cudaGetLastError();
}

cudaError_t launch_fused_pt(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                            const CUtensorMap& mapH, const CUtensorMap& mapZ, const FusedArgs& a, int D, int nsm,
                            cudaStream_t s) {
  return D == 128 ? launch_fused_pt_t<128>(mapQ, mapK, mapV, mapH, mapZ, a, nsm, s)
                  : launch_fused_pt_t<64>(mapQ, mapK, mapV, mapH, mapZ, a, nsm, s);
}

}  // namespace sla
