// Fused SLA / SLA2 forward, one tile per CTA walked by two softmax warpgroups
// ("SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
// Sparse-Linear Attention", §2 Q2 steps 3-4 and Fig. 4 "Fused kernel"; "SLA2:
// Sparse-Linear Attention with Learnable Routing and QAT", §3), bf16 Q K^T and
// P V.
//
// A tile is 128 query rows = two query blocks of one head (paired for
// overlapping critical lists) and walks the union of their critical lists two
// key blocks per step: S = Q [K_j; K_j']^T is one N = 128 MMA, O += P [V_j; V_j']
// one K = 128 chain.  The steps alternate between two slots, each with its own
// score buffer, O accumulator and softmax warpgroup (split of the key set: slot
// A takes steps 0, 2, 4, ..., slot B steps 1, 3, 5, ...), so while one slot's
// warpgroup computes its softmax the tensor cores run the other slot's products,
// and the MMA warp issues in the fixed order S_0, S_1, PV_0, S_2, PV_1, S_3, ...
// At the end of the tile the two slots' running maxima and sums are exchanged
// through TMEM and merged:
//     O = c_A O_A + c_B O_B,  c_X = w_s 2^(m_X - M),  M = max(m_A, m_B),
//     l = l_A 2^(m_A - M) + l_B 2^(m_B - M),  w_s = 1 / l (SLA) or a / l (SLA2).
// The linear branch is folded into O_A: P' = phi~(q) w_l / c_A goes into TMEM and
// the MMA warp adds P'_a H_a^T + P'_b H_b^T (one chain per query block, the
// other half's rows zero), w_l = 1 / den (SLA) or (1 - a) / den (SLA2), with
// phi~(q) H / (phi~(q) Z + s eps) = phi(q) H / (phi(q) Z + eps) exactly.
//
// K, V and H tiles stream through one ring of 32 KB stages (two key blocks of K
// or of V, or one H tile) in the MMA warp's consumption order, so the loads run
// several steps ahead.  CTAs are persistent (one per SM) and take tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...
//
//   warp 0      TMA producer: union record, Q tile, then the ring
//   warp 1      MMA issuer
//   warps 2-5   slot A's softmax (one query row per thread), then phi~(q), P'
//               and half of the epilogue's columns
//   warps 6-9   slot B's softmax, then the other half of the columns
//
// TMEM: S_A [0, 128), S_B [128, 256), O_A [256, 256 + d), O_B [384, 384 + d).
// Each slot's running (m, l) is exchanged through columns 64, 65 of its own
// score buffer; P'_a goes into S_A columns [0, d/2), P'_b into S_B [0, d/2).
#include "kernels.cuh"

namespace sla {

namespace {

constexpr float SK_RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr float SK_LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float sk_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct SkSmem {
  static constexpr int CH = D / 64;              // 64-column chunks of d
  static constexpr int Q_BYTES = 128 * D * 2;    // [chunk][128 rows][128 B]
  static constexpr int KT_BYTES = 64 * D * 2;    // one key block of K or V
  static constexpr int ST_BYTES = 2 * KT_BYTES;  // a ring stage: two key blocks, or one H tile
  static constexpr int NS = 6;                   // ring stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_R = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_R + NS * ST_BYTES;
  static constexpr int OFF_U = OFF_BAR + 256;    // two union records
  static size_t bytes(int urec_bytes) { return (size_t)OFF_U + 2 * (size_t)urec_bytes + 1024; }
};
static_assert(SkSmem<128>::ST_BYTES >= 128 * 128 * 2 && SkSmem<64>::ST_BYTES >= 64 * 64 * 2,
              "an H tile must fit a ring stage");

// One softmax step of one query row over the S columns of the step's key
// blocks: ne (1 or 2) blocks, block e critical for this row's query block when
// bit e of `crit` is set, nv[e] its real tokens.  Compact on purpose (the two
// warpgroups run it at different places, and a fully unrolled 128-column body
// per case overflows the instruction cache): the 32-column chunks are loaded
// from TMEM twice, once for the row max and once for the exponentials.  Writes P
// (bf16 pairs, keys 2c and 2c + 1 in column c; zeros for a block that is not
// critical) over the first 32 * ne columns of S, then rescales O if the max grew
// by more than the threshold (O must first hold the slot's previous P V).
// Returns false if a wait gave up.
template <int D>
__device__ __noinline__ bool sk_softmax_step(uint32_t tS, uint32_t tO, int ne, uint32_t crit, int nv0, int nv1,
                                             float sl2, float& m, float& l, uint64_t* pv_prev,
                                             uint32_t pv_parity, int* err) {
  float mx = -INFINITY;
#pragma unroll 1
  for (int q = 0; q < 2 * ne; ++q) {
    if (!((crit >> (q >> 1)) & 1u)) continue;  // warp-uniform
    uint32_t sv[32];
    tmem_ld32(tS + 32 * q, sv);
    tmem_ld_wait();
    const int nv = ((q >> 1) ? nv1 : nv0) - 32 * (q & 1);  // real tokens from this chunk's first column
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (c < nv) mx = fmaxf(mx, __uint_as_float(sv[c]));
  }
  bool grow = false;
  float fsc = 1.f;
  if (crit) {
    mx *= sl2;
    const bool first = (m == -INFINITY);
    grow = !first && (mx - m > SK_RESCALE_THRESHOLD);
    if (first) m = mx;  // O and l of this row are still exactly 0 in this slot
    if (grow) {
      fsc = sk_ex2(m - mx);
      m = mx;
    }
  }
  const float nm = -m;
  float lsum = 0.f;
#pragma unroll 1
  for (int q = 0; q < 2 * ne; ++q) {
    if (!((crit >> (q >> 1)) & 1u)) {
      tmem_st16_zero(tS + 16 * q);
      continue;
    }
    uint32_t sv[32], pk[16];
    tmem_ld32(tS + 32 * q, sv);
    tmem_ld_wait();
    const int nv = ((q >> 1) ? nv1 : nv0) - 32 * (q & 1);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float p0 = 2 * c < nv ? sk_ex2(fmaf(__uint_as_float(sv[2 * c]), sl2, nm)) : 0.f;
      const float p1 = 2 * c + 1 < nv ? sk_ex2(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, nm)) : 0.f;
      lsum += p0 + p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    // P of chunk q over columns [16 q, 16 q + 16), whose scores have been read already
    tmem_st16(tS + 16 * q, pk);
  }
  l = l * fsc + lsum;
  if (__any_sync(0xffffffffu, grow)) {
    // the slot's next P V waits for this step's p_ready, so O is not written meanwhile
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

}  // namespace

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(320, 1)
    sla_fused_sk_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapH,
                        FusedArgs a) {
  using L = SkSmem<D>;
  constexpr int CH = L::CH, NS = L::NS, KT = L::KT_BYTES, ST = L::ST_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sR = sm + L::OFF_R;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_free = bars + 1;
  uint64_t* r_full = bars + 2;          // [NS]
  uint64_t* r_empty = r_full + NS;      // [NS]
  uint64_t* s_full = r_empty + NS;      // [2] per slot
  uint64_t* p_ready = s_full + 2;       // [2]
  uint64_t* pv_done = p_ready + 2;      // [2]
  uint64_t* ml_ready = pv_done + 2;
  uint64_t* lin_ready = ml_ready + 1;
  uint64_t* o_full = lin_ready + 1;
  uint64_t* o_free = o_full + 1;
  uint64_t* u_full = o_free + 1;        // [2]
  uint64_t* u_free = u_full + 2;        // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(u_free + 2);
  const int urec = a.urec;
  uint16_t* sU = reinterpret_cast<uint16_t*>(sm + L::OFF_U);

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int npair = (a.Tq + 1) / 2;
  const int ntiles = a.BH * npair;

  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 4);
    for (int x = 0; x < NS; ++x) {
      mbar_init(&r_full[x], 1);
      mbar_init(&r_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[x], 4);
      mbar_init(&pv_done[x], 1);
      mbar_init(&u_full[x], 1);
      mbar_init(&u_free[x], 9);
    }
    mbar_init(ml_ready, 8);
    mbar_init(lin_ready, 8);
    mbar_init(o_full, 1);
    mbar_init(o_free, 8);
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
      uint32_t fill = 0;  // ring fills so far (stage = fill % NS)
      bool ok = true;
      auto claim = [&](uint32_t bytes) -> int {
        const int st = (int)(fill % NS);
        if (fill >= (uint32_t)NS && !mbar_wait(&r_empty[st], ((fill / NS) - 1) & 1, a.err, DEV_TIMEOUT_SYNC))
          return -1;
        mbar_arrive_expect_tx(&r_full[st], bytes);
        return st;
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
        // Q tile (the previous tile's phi~(q) has been read from sQ)
        if (it >= 1 && !mbar_wait(q_free, (it - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        mbar_arrive_expect_tx(q_full, L::Q_BYTES);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          tma_load_4d(sQ + c * 16384, &mapQ, q_full, c * 64, 64 * ia, h, b);
          tma_load_4d(sQ + c * 16384 + 8192, &mapQ, q_full, c * 64, 64 * ibl, h, b);
        }
        if (!mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) break;
        const int U = u[0];
        const int nst = (U + 1) / 2;
        // K pair of step s: [chunk c][key block e][64 rows][128 B]
        auto load_k = [&](int s) -> bool {
          const int ne = (2 * s + 1 < U) ? 2 : 1;
          const int st = claim(ne * KT);
          if (st < 0) return false;
          for (int e = 0; e < ne; ++e) {
            const int j = u[8 + 2 * s + e] & 0x3fff;
#pragma unroll
            for (int c = 0; c < CH; ++c)
              tma_load_4d(sR + st * ST + c * 16384 + e * 8192, &mapK, &r_full[st], c * 64, 64 * j, h, b);
          }
          ++fill;
          return true;
        };
        // V pair of step s: [key block e][chunk c][64 rows][128 B]
        auto load_v = [&](int s) -> bool {
          const int ne = (2 * s + 1 < U) ? 2 : 1;
          const int st = claim(ne * KT);
          if (st < 0) return false;
          for (int e = 0; e < ne; ++e) {
            const int j = u[8 + 2 * s + e] & 0x3fff;
#pragma unroll
            for (int c = 0; c < CH; ++c)
              tma_load_4d(sR + st * ST + e * KT + c * 8192, &mapV, &r_full[st], c * 64, 64 * j, h, b);
          }
          ++fill;
          return true;
        };
        // the MMA warp's order: S_0, S_1, then PV_s, S_{s+2} for s = 0, 1, ...
        ok = load_k(0);
        if (ok && nst > 1) ok = load_k(1);
        for (int s = 0; s < nst && ok; ++s) {
          ok = load_v(s);
          if (ok && s + 2 < nst) ok = load_k(s + 2);
        }
        // H_a^T, then H_b^T
        for (int t = 0; t < 2 && ok; ++t) {
          const int st = claim(D * D * 2);
          if (st < 0) { ok = false; break; }
#pragma unroll
          for (int c = 0; c < CH; ++c)
            tma_load_4d(sR + st * ST + c * (D * 128), &mapH, &r_full[st], c * 64, 0, t == 0 ? ia : ibl, bh);
          ++fill;
        }
      }
    }
  } else if (w == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (ln == 0) {
      const uint32_t id_s128 = idesc_bf16(128, 128, false, false);
      const uint32_t id_s64 = idesc_bf16(128, 64, false, false);
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      const uint32_t id_l = idesc_bf16(128, D, false, false);
      const uint32_t q0 = smem_u32(sQ), r0 = smem_u32(sR);
      uint32_t use = 0;             // ring uses so far
      uint32_t gs[2] = {0u, 0u};    // steps per slot so far
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const int ub = it & 1;
        if (!mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA)) break;
        const int U = sU[ub * urec];
        const int nst = (U + 1) / 2;
        if (!mbar_wait(q_full, it & 1, a.err, DEV_TIMEOUT_TMA)) break;
        auto issue_s = [&](int s) -> bool {
          const int x = s & 1;
          const int st = (int)(use % NS);
          if (!mbar_wait(&r_full[st], (use / NS) & 1, a.err, DEV_TIMEOUT_TMA)) return false;
          tc_fence_after();
          const uint32_t kt = r0 + st * ST;
          const uint32_t id = (2 * s + 1 < U) ? id_s128 : id_s64;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(q0 + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kt + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
            umma_ss(tbase + 128 * x, ad, bd, id, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[x]);
          umma_commit(&r_empty[st]);
          ++use;
          return true;
        };
        auto issue_pv = [&](int s) -> bool {
          const int x = s & 1;
          const bool first = s < 2;  // the slot's first step of this tile
          if (!mbar_wait(&p_ready[x], gs[x] & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
          // the previous tile's epilogue must have read O before it is overwritten
          if (first && it > 0 && !mbar_wait(o_free, (it - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
          const int st = (int)(use % NS);
          if (!mbar_wait(&r_full[st], (use / NS) & 1, a.err, DEV_TIMEOUT_TMA)) return false;
          tc_fence_after();
          const uint32_t vt = r0 + st * ST;
          const int nk = (2 * s + 1 < U) ? 8 : 4;
          for (int kk = 0; kk < nk; ++kk)
            umma_ts(tbase + 256 + 128 * x, tbase + 128 * x + 8 * kk,
                    sdesc_sw128(vt + (kk / 4) * KT + (kk % 4) * 2048, 8192, 1024), id_pv,
                    (!first || kk > 0) ? 1u : 0u);
          umma_commit(&pv_done[x]);
          umma_commit(&r_empty[st]);
          ++use;
          ++gs[x];
          return true;
        };
        ok = issue_s(0);
        if (ok && nst > 1) ok = issue_s(1);
        for (int s = 0; s < nst && ok; ++s) {
          ok = issue_pv(s);
          if (ok && s + 2 < nst) ok = issue_s(s + 2);
        }
        if (!ok) break;
        // linear branch: O_A += P'_a H_a^T + P'_b H_b^T
        if (!mbar_wait(lin_ready, it & 1, a.err, DEV_TIMEOUT_SYNC)) break;
        for (int t = 0; t < 2 && ok; ++t) {
          const int st = (int)(use % NS);
          if (!mbar_wait(&r_full[st], (use / NS) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ht = r0 + st * ST;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ts(tbase + 256, tbase + 128 * t + 8 * kk,
                    sdesc_sw128(ht + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024), id_l, 1u);
          umma_commit(&r_empty[st]);
          ++use;
        }
        if (!ok) break;
        umma_commit(o_full);
        mbar_arrive(&u_free[ub]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int X = (w - 2) >> 2;  // slot: 0 (warps 2-5) or 1 (warps 6-9)
    const int q4 = w & 3;
    const int r = 32 * q4 + ln;
    const int half = r >> 6;
    const uint32_t bit = 1u << half;
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const uint32_t tS = tbase + 128 * X + lane_off;        // this slot's score buffer
    const uint32_t tO = tbase + 256 + 128 * X + lane_off;  // this slot's O
    const uint32_t tSo = tbase + 128 * (1 - X) + lane_off; // the other slot's score buffer
    const uint32_t tOA = tbase + 256 + lane_off, tOB = tbase + 384 + lane_off;
    const float sl2 = a.scale_log2;
    uint32_t g = 0;  // this slot's steps so far
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const int ub = it & 1;
      const uint16_t* u = sU + ub * urec;
      if (!__all_sync(0xffffffffu, mbar_wait(&u_full[ub], (it >> 1) & 1, a.err, DEV_TIMEOUT_TMA))) break;
      const int U = u[0];
      const int nst = (U + 1) / 2;
      const int bh = tile / npair, p = tile % npair;
      const int2 pr = a.pairs[(int64_t)bh * npair + p];
      const bool has_b = pr.y >= 0;
      const int blk = half == 0 ? pr.x : (has_b ? pr.y : pr.x);
      const float alpha = a.combine == 1 ? a.alpha[bh] : 1.f;
      const bool sparse_on = alpha != 0.f;  // SLA2 with alpha = 0: only the linear branch
      float m = -INFINITY, l = 0.f;
      for (int s = X; s < nst; s += 2, ++g) {
        const bool two = 2 * s + 1 < U;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[X], g & 1, a.err, DEV_TIMEOUT_MMA))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t f0 = u[8 + 2 * s], f1 = two ? u[9 + 2 * s] : 0u;
        const bool c0 = sparse_on && ((f0 >> 14) & bit);  // warp-uniform
        const bool c1 = sparse_on && two && ((f1 >> 14) & bit);
        const int nv0 = a.N - 64 * (int)(f0 & 0x3fff), nv1 = a.N - 64 * (int)(f1 & 0x3fff);
        const bool good = sk_softmax_step<D>(tS, tO, two ? 2 : 1, (c0 ? 1u : 0u) | (c1 ? 2u : 0u), nv0, nv1, sl2,
                                             m, l, &pv_done[X], (g - 1) & 1, a.err);
        if (!good) {
          ok = false;
          break;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (ln == 0) mbar_arrive(&p_ready[X]);
      }
      if (!ok) break;
      // ---------------- merge the two slots: (m, l) through columns 64, 65 of each score buffer
      const bool had = nst > X;  // this slot ran at least one step of the tile
      if (had) ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[X], (g - 1) & 1, a.err, DEV_TIMEOUT_MMA));
      if (!ok) break;
      tc_fence_after();
      tmem_st2(tS + 64, __float_as_uint(m), __float_as_uint(l));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (ln == 0) mbar_arrive(ml_ready);
      if (!__all_sync(0xffffffffu, mbar_wait(ml_ready, it & 1, a.err, DEV_TIMEOUT_SYNC))) { ok = false; break; }
      tc_fence_after();
      uint32_t mo_u, lo_u;
      tmem_ld2(tSo + 64, mo_u, lo_u);
      tmem_ld_wait();
      const float mA = X == 0 ? m : __uint_as_float(mo_u), lA = X == 0 ? l : __uint_as_float(lo_u);
      const float mB = X == 1 ? m : __uint_as_float(mo_u), lB = X == 1 ? l : __uint_as_float(lo_u);
      const float M = fmaxf(mA, mB);
      const float eA = M == -INFINITY ? 0.f : sk_ex2(mA - M), eB = M == -INFINITY ? 0.f : sk_ex2(mB - M);
      const float lt = lA * eA + lB * eB;
      const float ws = (lt > 0.f) ? alpha / lt : 0.f;  // alpha = 1 for SLA
      const float cA = ws * eA > 0.f ? ws * eA : 1.f, cB = ws * eB;
      const int n = 64 * blk + (r & 63);
      const bool store = (n < a.N) && (half == 0 || has_b);
      constexpr int HC = D / 2;  // this warpgroup's columns of the epilogue: [HC X, HC X + HC)
      if (a.lse || a.os) {
        // for the backward: the sparse branch alone (O_A, O_B hold only P V so far) and
        // the log-sum-exp of the row's scaled critical scores, sum_t exp(s_t) = 2^M l
        const float inv_l = (lt > 0.f) ? 1.f / lt : 0.f;
        if (a.lse && store && X == 0) a.lse[(int64_t)bh * a.N + n] = (M + log2f(lt)) * 0.6931471805599453f;
        if (a.os) {
#pragma unroll 1
          for (int c0 = HC * X; c0 < HC * X + HC; c0 += 32) {
            uint32_t oa[32], ob[32];
            tmem_ld32(tOA + c0, oa);
            tmem_ld32(tOB + c0, ob);
            tmem_ld_wait();
            if (store) {
              float4* od = reinterpret_cast<float4*>(a.os + ((int64_t)bh * a.N + n) * D + c0);
              float y[32];
#pragma unroll
              for (int c = 0; c < 32; ++c)
                y[c] = (__uint_as_float(oa[c]) * eA + (eB != 0.f ? __uint_as_float(ob[c]) * eB : 0.f)) * inv_l;
#pragma unroll
              for (int v = 0; v < 8; ++v) od[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
            }
          }
        }
      }
      if (X == 0) {
        // ---------------- linear branch: P' = phi~(q_r) * (w_l / c_A), e = phi~(q) as bf16 pairs
        if (!__all_sync(0xffffffffu, mbar_wait(q_full, it & 1, a.err, DEV_TIMEOUT_TMA))) { ok = false; break; }
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
          const float nmq = -mq * SK_LOG2E;
          const uint4* zrow = reinterpret_cast<const uint4*>(a.Hz + ((int64_t)bh * a.Tq + blk) * a.NN + D * D);
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const uint4 zv = __ldg(zrow + c8);
            const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(&zv);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const int c = 4 * c8 + e2;
              const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
              const float x0 = __low2float(q2), x1 = __high2float(q2);
              const float e0 = elu ? (x0 > 0.f ? x0 + 1.f : sk_ex2(x0 * SK_LOG2E)) : sk_ex2(fmaf(x0, SK_LOG2E, nmq));
              const float e1 = elu ? (x1 > 0.f ? x1 + 1.f : sk_ex2(x1 * SK_LOG2E)) : sk_ex2(fmaf(x1, SK_LOG2E, nmq));
              pe[c] = pack_bf16x2(e0, e1);
              const __nv_bfloat162 eb = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
              esum += __low2float(eb) + __high2float(eb);
              edotz = fmaf(__low2float(eb), __low2float(z2[e2]), fmaf(__high2float(eb), __high2float(z2[e2]), edotz));
            }
          }
          if (elu) esum = 1.f;
        }
        // sQ has been read: the producer may load the next tile's Q
        __syncwarp();
        if (ln == 0) mbar_arrive(q_free);
        const float den = edotz + esum * a.eps;
        const float wl = (a.combine == 1 ? 1.f - alpha : 1.f) / den;
        const float pscale = wl / cA;
#pragma unroll
        for (int c = 0; c < D / 2; ++c) {
          const __nv_bfloat162 eb = *reinterpret_cast<const __nv_bfloat162*>(&pe[c]);
          pe[c] = pack_bf16x2(__low2float(eb) * pscale, __high2float(eb) * pscale);
        }
        // P'_a into S_A [0, D/2), P'_b into S_B [0, D/2): this row's half carries phi~(q)
        const uint32_t tSA = tbase + lane_off, tSB = tbase + 128 + lane_off;
#pragma unroll
        for (int c0p = 0; c0p < D / 2; c0p += 32) {
          uint32_t chunk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) chunk[c] = pe[c0p + c];
          tmem_st32((half == 0 ? tSA : tSB) + c0p, chunk);
          tmem_st32_zero((half == 0 ? tSB : tSA) + c0p);
        }
        tmem_st_wait();
      }
      // (m, l) read, O^s stored: the MMA warp may add the linear term and reuse the score buffers
      tc_fence_before();
      __syncwarp();
      if (ln == 0) mbar_arrive(lin_ready);
      // ---------------- epilogue: c_A O_A + c_B O_B (+ bias), this warpgroup's half of the columns
      if (!__all_sync(0xffffffffu, mbar_wait(o_full, it & 1, a.err, DEV_TIMEOUT_MMA))) { ok = false; break; }
      tc_fence_after();
      {
        const int b = bh / a.H, h = bh % a.H;
        __nv_bfloat16* orow = a.O + (int64_t)b * a.so0 + (int64_t)h * a.so1 + (int64_t)n * a.so2;
#pragma unroll 1
        for (int c0 = HC * X; c0 < HC * X + HC; c0 += 32) {
          uint32_t oa[32], ob[32];
          tmem_ld32(tOA + c0, oa);
          tmem_ld32(tOB + c0, ob);
          tmem_ld_wait();
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int c = 8 * v + e;
                const float bias = (a.combine == 0 && a.proj_b) ? __ldg(a.proj_b + c0 + c) : 0.f;
                y[e] = __uint_as_float(oa[c]) * cA + (cB != 0.f ? __uint_as_float(ob[c]) * cB : 0.f) + bias;
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
    tmem_dealloc(tbase, 512);
  }
}

size_t fused_sk_smem_bytes(int D, int urec) {
  return D == 128 ? SkSmem<128>::bytes(urec * 2) : SkSmem<64>::bytes(urec * 2);
}

template <int D>
static cudaError_t launch_fused_sk_t(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                     const CUtensorMap& mapH, const FusedArgs& a, int nsm, cudaStream_t s) {
  const size_t smem = SkSmem<D>::bytes(a.urec * 2);
  cudaError_t e = cudaFuncSetAttribute(sla_fused_sk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntiles = a.BH * ((a.Tq + 1) / 2);
  const int grid = ntiles < nsm ? ntiles : nsm;
  sla_fused_sk_kernel<D><<<grid, 320, smem, s>>>(mapQ, mapK, mapV, mapH, a);
  return cudaGetLastError();
}

cudaError_t launch_fused_sk(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                            const CUtensorMap& mapH, const FusedArgs& a, int D, int nsm, cudaStream_t s) {
  return D == 128 ? launch_fused_sk_t<128>(mapQ, mapK, mapV, mapH, a, nsm, s)
                  : launch_fused_sk_t<64>(mapQ, mapK, mapV, mapH, a, nsm, s);
}

}  // namespace sla
