// Fused SLA / SLA2 forward for one pair of query blocks ("SLA: Beyond
// Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
// Attention", §2 Q2 steps 3-4 and Fig. 4 "Fused kernel"; "SLA2: Sparse-Linear
// Attention with Learnable Routing and QAT", §3).
//
// A CTA owns 128 query rows = two query blocks of one head (chosen by
// pairing_kernel for similar critical lists), so every tcgen05.mma runs at
// M = 128.  It walks the union of the two blocks' critical lists (ascending); a
// key block that is critical for only one of the two query blocks is masked out
// of the other half (its probabilities are 0).
//
//   warp 0      TMA producer: Q tile, then K_j and V_j per union entry through
//               two separate rings (a K slot frees when its S MMA completes, a
//               V slot when its P V completes, so K tiles run ahead), then the
//               aggregated H_i^T tiles and Z_i rows (H_a into the K ring, H_b
//               into the V ring)
//   warp 1      MMA issuer: S_k = Q K_j^T into TMEM (two buffers), O += P_k V_j
//               with P_k read back from TMEM, and at the end
//               L = phi~(Q) H_i^T for both query blocks
//   warps 2-5   one query row per thread: online softmax with exp2 (lazy
//               rescale of O in TMEM only when the running max grows by more
//               than 2^8), P_k written over S_k; after the loop phi~(Q)
//               (unnormalised softmax of q over d) in place of Q, then the
//               combine  O = O^s + O^l (+ bias)  or  a O^s + (1 - a) O^l.
//
// Resources are sized for two co-resident CTAs per SM (256 TMEM columns,
// about 100 KB of shared memory), so one CTA's softmax, prologue and epilogue
// overlap the other CTA's tensor-core work.
//
// TMEM columns: S0 [0,64) (P0 over its first 32 columns), S1 [64,128) (P1),
// O [128,128+d).  After the last P V the S/P region [0,d) holds L_a; once the
// rows of query block 2p have been written out it holds L_b.
//
// Low-bit variant ([SLA2] §5): Q and K arrive as 8-bit codes (E4M3, or
// symmetric INT8) with one scale per (head, 64-row block) and S = Q^ K^^T runs
// as tcgen05.mma kind::f8f6f4 (fp32 accumulate) or kind::i8 (int32 accumulate);
// the softmax multiplies the scores by s_Q s_K.  The 8-bit Q tile and K ring are
// half the size, so the bf16 Q tile (needed for phi(Q)) fits beside them and
// H_a loads over the 8-bit Q tile and K ring.
//
// Linear branch with unnormalised feature map: for e_a = 2^((q_a - max q) log2 e)
// and s = sum_a e_a, phi(q) = e / s, so
//     phi(q) H / (phi(q) Z + eps) = (e H) / (e Z + s eps)      exactly.
// With the elu + 1 feature map ([SLA] Table 2 ablation) e = phi(q) and s = 1.
//
// FP8 P V (PV8, [SLA2] §5: P and V quantised, their product dequantised): V
// arrives as E4M3 with one scale per (head, channel), transposed per key block
// ([d rows][64 tokens, padded to 128 B]: the K-major B operand); the running
// maximum is kept in whole log2 units and raised on every increase (no lazy
// rescale), so P <= 1, every rescale of O is an exact power of two, and
// P^ = E4M3(448 P) is written over S (four values per TMEM column); O += P^ V^
// runs as kind::f8f6f4 with P^ read from TMEM, and the epilogue applies
// s_V[c] / 448.  The row sum l uses the unquantised P.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace sla {

template <int D, bool FP8>
struct FusedSmem {
  static constexpr int CH = D / 64;
  static constexpr int NR = (D == 128) ? 2 : 4;        // slots per ring (K ring and V ring)
  static constexpr int Q_BYTES = 128 * D * 2;          // bf16 Q tile
  static constexpr int Q8_BYTES = FP8 ? 128 * D : 0;   // e4m3 Q tile
  static constexpr int KT_BYTES = 64 * D * 2;          // one bf16 K or V tile
  static constexpr int KSLOT = FP8 ? 64 * D : KT_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_Q8 = OFF_Q + Q_BYTES;
  static constexpr int OFF_K = OFF_Q8 + Q8_BYTES;
  static constexpr int OFF_V = OFF_K + NR * KSLOT;
  static constexpr int OFF_HA = FP8 ? OFF_Q8 : OFF_K;  // H_a goes where Q8 / K were
  static constexpr int OFF_Z = OFF_V + NR * KT_BYTES;  // Z_a, Z_b: 2 x D bf16 (unswizzled rows)
  static constexpr int OFF_BAR = OFF_Z + 2 * CH * 128;
  static constexpr int OFF_U = OFF_BAR + 256;
  static size_t bytes(int Tkv) { return (size_t)OFF_U + 9 * (size_t)((Tkv + 15) & ~15) + 1024; }
};
static_assert(FusedSmem<128, false>::OFF_V - FusedSmem<128, false>::OFF_HA >= 128 * 128 * 2 &&
                  FusedSmem<128, true>::OFF_V - FusedSmem<128, true>::OFF_HA >= 128 * 128 * 2 &&
                  FusedSmem<64, false>::OFF_V - FusedSmem<64, false>::OFF_HA >= 64 * 64 * 2,
              "an H tile must fit where it is loaded");
static_assert(FusedSmem<128, false>::NR * FusedSmem<128, false>::KT_BYTES >= 128 * 128 * 2,
              "H_b must fit the V ring");

namespace {
constexpr uint32_t COL_S = 0, COL_O = 128, COL_L = 0;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^n for a whole number n <= 0, exactly (0 below the normal range)
__device__ __forceinline__ float exp2_whole(float n) {
  const int e = 127 + __float2int_rn(n);
  return e > 0 ? __int_as_float(e << 23) : 0.f;
}

}  // namespace

template <int D, int QK8, bool PV8>
__global__ void __launch_bounds__(192, 2)
    sla_fused_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                     const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapH,
                     const __grid_constant__ CUtensorMap mapZ, const __grid_constant__ CUtensorMap mapQ8,
                     const __grid_constant__ CUtensorMap mapK8, FusedArgs a) {
  constexpr bool FP8 = QK8 != 0;  // 8-bit Q K^T: 1 E4M3 (kind::f8f6f4), 2 INT8 (kind::i8)
  static_assert(!FP8 || D == 128, "the 8-bit Q K^T path is built for d = 128");
  static_assert(!PV8 || D == 128, "the FP8 P V path is built for d = 128");
  using L = FusedSmem<D, FP8>;
  constexpr int NR = L::NR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sQ8 = sm + L::OFF_Q8;
  uint8_t* sK = sm + L::OFF_K;
  uint8_t* sV = sm + L::OFF_V;
  uint8_t* sHa = sm + L::OFF_HA;
  uint8_t* sZ = sm + L::OFF_Z;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* phiq_ready = bars + 1;
  uint64_t* la_full = bars + 2;
  uint64_t* lb_full = bars + 3;
  uint64_t* la_free = bars + 4;
  uint64_t* s_full = bars + 5;     // [2]
  uint64_t* p_ready = bars + 7;    // [2]
  uint64_t* pv_done = bars + 9;    // [2]
  uint64_t* ha_full = bars + 11;
  uint64_t* hb_full = bars + 12;
  uint64_t* k_full = bars + 13;    // [NR]
  uint64_t* k_empty = k_full + NR;
  uint64_t* v_full = k_empty + NR;
  uint64_t* v_empty = v_full + NR;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(v_empty + NR);
  int* s_count = reinterpret_cast<int*>(tslot + 1);
  const int Tkvr = (a.Tkv + 15) & ~15;
  uint8_t* fa = sm + L::OFF_U;
  uint8_t* fb = fa + Tkvr;
  uint8_t* uflag = fb + Tkvr;
  uint16_t* uidx = reinterpret_cast<uint16_t*>(uflag + Tkvr);
  float* usk = reinterpret_cast<float*>(uidx + Tkvr);  // FP8: K scale per union entry

  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int p = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  // the CTA's two query blocks (rows 0-63: ia, rows 64-127: ib); ib < 0: none
  const int2 pair = a.pairs[(int64_t)bh * ((a.Tq + 1) / 2) + p];
  const int ia = pair.x, ib = pair.y;
  const bool has_b = ib >= 0;
  const int ibl = has_b ? ib : ia;  // block loaded into the second half

  // ---------------- set-up: TMEM, barriers, union of the two critical lists
  if (w == 1) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(phiq_ready, 128);
    mbar_init(la_full, 1);
    mbar_init(lb_full, 1);
    mbar_init(la_free, 64);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[x], 128);
      mbar_init(&pv_done[x], 1);
    }
    mbar_init(ha_full, 1);
    mbar_init(hb_full, 1);
    for (int s = 0; s < NR; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    fence_barrier_init();
  }
  for (int j = tid; j < 2 * Tkvr; j += blockDim.x) fa[j] = 0;  // fa and fb
  __syncthreads();
  {
    const int32_t* la = a.lut + ((int64_t)bh * a.Tq + ia) * a.nh;
    const int32_t* lb = a.lut + ((int64_t)bh * a.Tq + (has_b ? ib : ia)) * a.nh;
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
        if (FP8) usk[pos] = a.scale_k[(int64_t)bh * a.Tkv + j];
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
    // ---------------- TMA producer
    if (ln == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      tma_prefetch_desc(&mapH);
      tma_prefetch_desc(&mapZ);
      if (FP8) tma_prefetch_desc(&mapQ8), tma_prefetch_desc(&mapK8);
      mbar_arrive_expect_tx(q_full, L::Q_BYTES + L::Q8_BYTES);
#pragma unroll
      for (int c = 0; c < L::CH; ++c) {
        tma_load_4d(sQ + c * 16384, &mapQ, q_full, c * 64, 64 * ia, h, b);
        tma_load_4d(sQ + c * 16384 + 8192, &mapQ, q_full, c * 64, 64 * ibl, h, b);
      }
      if (FP8) {
        tma_load_3d(sQ8, &mapQ8, q_full, 0, 64 * ia, bh);
        tma_load_3d(sQ8 + 8192, &mapQ8, q_full, 0, 64 * ibl, bh);
      }
      bool ok = true;
      // K_k is issued one step ahead of V_{k-1}
      for (int k = 0; k <= U && ok; ++k) {
        if (k < U) {
          const int s = k % NR;
          if (k >= NR && !mbar_wait(&k_empty[s], ((k / NR) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
            ok = false;
            break;
          }
          const int j = uidx[k];
          mbar_arrive_expect_tx(&k_full[s], L::KSLOT);
          if (FP8) {
            tma_load_3d(sK + s * L::KSLOT, &mapK8, &k_full[s], 0, 64 * j, bh);
          } else {
#pragma unroll
            for (int c = 0; c < L::CH; ++c)
              tma_load_4d(sK + s * L::KSLOT + c * 8192, &mapK, &k_full[s], c * 64, 64 * j, h, b);
          }
        }
        if (k >= 1) {
          const int kv = k - 1, s = kv % NR;
          if (kv >= NR && !mbar_wait(&v_empty[s], ((kv / NR) - 1) & 1, a.err, DEV_TIMEOUT_SYNC)) {
            ok = false;
            break;
          }
          const int j = uidx[kv];
          mbar_arrive_expect_tx(&v_full[s], L::KT_BYTES);
          if (PV8) {  // V^ of block j: [d rows][128 B], the same 16 KB as a bf16 V tile
            tma_load_3d(sV + s * L::KT_BYTES, &mapV, &v_full[s], 0, D * j, bh);
          } else {
#pragma unroll
            for (int c = 0; c < L::CH; ++c)
              tma_load_4d(sV + s * L::KT_BYTES + c * 8192, &mapV, &v_full[s], c * 64, 64 * j, h, b);
          }
        }
      }
      // H_a (+ Z_a) into the K ring once its last S MMAs completed, H_b (+ Z_b)
      // into the V ring once its last P V completed
      for (int t = 0; t < 2 && ok; ++t) {
        uint64_t* empty = (t == 0) ? k_empty : v_empty;
        for (int s = 0; s < NR && ok; ++s) {
          if (U > s) {
            const int last = s + NR * ((U - 1 - s) / NR);
            ok = mbar_wait(&empty[s], (last / NR) & 1, a.err, DEV_TIMEOUT_SYNC);
          }
        }
        if (!ok) break;
        const int i = (t == 0) ? ia : (has_b ? ib : ia);
        uint64_t* full = (t == 0) ? ha_full : hb_full;
        uint8_t* dst = (t == 0) ? sHa : sV;
        mbar_arrive_expect_tx(full, D * D * 2 + D * 2);
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_load_4d(dst + c * (D * 128), &mapH, full, c * 64, 0, i, bh);
          tma_load_3d(sZ + (t * L::CH + c) * 128, &mapZ, full, D * D + c * 64, i, bh);
        }
      }
    }
  } else if (w == 1) {
    // ---------------- MMA issuer
    if (ln == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_s8 = QK8 == 2 ? idesc_s8(128, 64) : idesc_e4m3(128, 64);
      const uint32_t id_pv = idesc_bf16(128, D, false, true);
      const uint32_t id_pv8 = idesc_e4m3(128, D);
      const uint32_t id_l = idesc_bf16(128, D, false, false);
      const uint32_t q0 = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, a.err, DEV_TIMEOUT_TMA);
      auto issue_pv = [&](int kp) -> bool {
        if (!mbar_wait(&p_ready[kp & 1], (kp >> 1) & 1, a.err, DEV_TIMEOUT_SYNC)) return false;
        const int sv = kp % NR;
        if (!mbar_wait(&v_full[sv], (kp / NR) & 1, a.err, DEV_TIMEOUT_TMA)) return false;
        tc_fence_after();
        const uint32_t vt = smem_u32(sV + sv * L::KT_BYTES);
        if (PV8) {
          // P^ (E4M3, 4 per column) from TMEM, V^ K-major: 32 tokens per instruction
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts_f8(tbase + COL_O, tbase + COL_S + 64 * (kp & 1) + 8 * kk, sdesc_sw128(vt + kk * 32, 16, 1024),
                       id_pv8, (kp > 0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_sw128(vt + kk * 2048, 8192, 1024);
            umma_ts(tbase + COL_O, tbase + COL_S + 64 * (kp & 1) + 8 * kk, bd, id_pv,
                    (kp > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&pv_done[kp & 1]);
        umma_commit(&v_empty[sv]);
        return true;
      };
      for (int k = 0; k < U && ok; ++k) {
        const int s = k % NR;
        if (!mbar_wait(&k_full[s], (k / NR) & 1, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
        // S buffer k&1 still holds P_{k-2}.  No wait is needed before
        // overwriting it: P_{k-2} V was issued earlier by this thread, and
        // tcgen05.mma operations issued by one thread execute in issue order.
        tc_fence_after();
        const uint32_t kt = smem_u32(sK + s * L::KSLOT);
        if (FP8) {
          // e4m3: 128-byte rows hold all d = 128 values; K = 32 per instruction
          const uint32_t q8 = smem_u32(sQ8);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t ad = sdesc_sw128(q8 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kt + kk * 32, 16, 1024);
            if (QK8 == 2)
              umma_ss_i8(tbase + COL_S + 64 * (k & 1), ad, bd, id_s8, kk > 0 ? 1u : 0u);
            else
              umma_ss_f8(tbase + COL_S + 64 * (k & 1), ad, bd, id_s8, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(q0 + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kt + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024);
            umma_ss(tbase + COL_S + 64 * (k & 1), ad, bd, id_s, kk > 0 ? 1u : 0u);
          }
        }
        umma_commit(&s_full[k & 1]);
        umma_commit(&k_empty[s]);
        if (k >= 1 && !issue_pv(k - 1)) { ok = false; break; }
      }
      if (ok && U >= 1) ok = issue_pv(U - 1);
      // linear branch: L = phi~(Q) H_i^T into the S/P region, first for query
      // block 2p, then (after its rows are written out) for 2p+1
      if (ok && U >= 1)
        ok = mbar_wait(&pv_done[(U - 1) & 1], ((U - 1) >> 1) & 1, a.err, DEV_TIMEOUT_MMA);
      if (ok) ok = mbar_wait(phiq_ready, 0, a.err, DEV_TIMEOUT_SYNC);
      for (int t = 0; t < 2 && ok; ++t) {
        if (!mbar_wait(t == 0 ? ha_full : hb_full, 0, a.err, DEV_TIMEOUT_TMA)) { ok = false; break; }
        if (t == 1 && !mbar_wait(la_free, 0, a.err, DEV_TIMEOUT_SYNC)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ht = smem_u32(t == 0 ? sHa : sV);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(q0 + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(ht + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024);
          umma_ss(tbase + COL_L, ad, bd, id_l, kk > 0 ? 1u : 0u);
        }
        umma_commit(t == 0 ? la_full : lb_full);
      }
    }
  } else {
    // ---------------- softmax / epilogue warps: one query row per thread
    const int q4 = w & 3;
    const int r = 32 * q4 + ln;
    const int half = r >> 6;
    const uint32_t bit = 1u << half;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    const float sl2 = a.scale_log2;
    const float sq_half = FP8 ? a.scale_q[(int64_t)bh * a.Tq + ((half == 1 && has_b) ? ib : ia)] : 1.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int k = 0; k < U; ++k) {
      const int sb = k & 1;
      const uint32_t ts = tl + COL_S + 64 * sb;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (k >> 1) & 1, a.err, DEV_TIMEOUT_MMA))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool crit = (uflag[k] & bit) != 0;  // uniform over the warp
      uint32_t pk[32];
      if (crit) {
        uint32_t s0[32], s1[32];
        tmem_ld32(ts, s0);
        tmem_ld32(ts + 32, s1);
        tmem_ld_wait();
        if (QK8 == 2) {  // int32 dot products of the INT8 codes (exact in fp32: |S| < 2^24)
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            s0[c] = __float_as_uint((float)(int)s0[c]);
            s1[c] = __float_as_uint((float)(int)s1[c]);
          }
        }
        const int nvalid = a.N - 64 * (int)uidx[k];
        if (nvalid < 64) {  // partial last key block: padding columns get -inf
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
          t[i] = fmax3(__uint_as_float(e < 32 ? s0[e] : s1[e - 32]),
                       __uint_as_float(e + 1 < 32 ? s0[e + 1] : s1[e + 1 - 32]),
                       __uint_as_float(e + 2 < 32 ? s0[e + 2] : s1[e + 2 - 32]));
        }
        t[21] = __uint_as_float(s1[31]);
#pragma unroll
        for (int i = 0; i < 7; ++i) t[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
        t[7] = t[21];
        t[0] = fmax3(t[0], t[1], t[2]);
        t[1] = fmax3(t[3], t[4], t[5]);
        // 8-bit scores carry the two block scales: s = (q^ . k^) s_Q s_K
        const float sc = FP8 ? sl2 * sq_half * usk[k] : sl2;
        const float mx = fmax3(t[0], t[1], fmaxf(t[6], t[7])) * sc;
        // lazy rescale: keep the running max unless it grows by more than 2^8.
        // FP8 P V: the running max is kept in whole log2 units (the row max
        // rounded up), so every rescale is an exact power of two and the final
        // E4M3(448 P) values do not depend on the order of the critical blocks.
        const float mt = PV8 ? ceilf(mx) : mx;
        const bool first = (m == -INFINITY);
        const bool grow = !first && (mt - m > (PV8 ? 0.f : RESCALE_THRESHOLD));
        if (first) m = mt;  // O and l of this row are still exactly 0
        if (__any_sync(0xffffffffu, grow)) {
          // O must hold P_{k-1} V_{k-1} before it is rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(k - 1) & 1], ((k - 1) >> 1) & 1, a.err,
                                                  DEV_TIMEOUT_MMA))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = grow ? (PV8 ? exp2_whole(m - mt) : ex2(m - mx)) : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tl + COL_O + c0, o);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
            tmem_st32(tl + COL_O + c0, o);
          }
          tmem_st_wait();
          if (grow) {
            l *= f;
            m = mt;
          }
        }
        // p = 2^(s sc - m): scaling in pairs (each rounded as fmaf), sums in pairs
        const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m, -m);
        uint64_t u2[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2, nm2), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s1[2 * c]), __uint_as_float(s1[2 * c + 1])), sc2, nm2), x2, x3);
          const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
          u2[c] = f2_add(f2_pack(p0, p1), f2_pack(p2, p3));
          if (PV8) {  // E4M3(448 p), four tokens per 32-bit column
            const __nv_fp8x2_storage_t a01 =
                __nv_cvt_float2_to_fp8x2(make_float2(448.f * p0, 448.f * p1), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t a23 =
                __nv_cvt_float2_to_fp8x2(make_float2(448.f * p2, 448.f * p3), __NV_SATFINITE, __NV_E4M3);
            pk[c] = (uint32_t)a01;        // tokens 2c, 2c+1
            pk[16 + c] = (uint32_t)a23;   // tokens 32+2c, 33+2c
          } else {
            pk[c] = pack_bf16x2(p0, p1);
            pk[16 + c] = pack_bf16x2(p2, p3);
          }
        }

#pragma unroll
        for (int st = 8; st >= 1; st >>= 1)
#pragma unroll
          for (int c = 0; c < st; ++c) u2[c] = f2_add(u2[c], u2[c + st]);
        float ul, uh;
        f2_unpack(u2[0], ul, uh);
        l += ul + uh;
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      if (PV8) {
        // pk[c] holds tokens 2c, 2c+1 in its low 16 bits (c < 32, token order);
        // TMEM column q takes tokens 4q .. 4q+3, lowest token in the lowest byte
        uint32_t p16[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) p16[q] = (pk[2 * q] & 0xffffu) | (pk[2 * q + 1] << 16);
        tmem_st16(ts, p16);  // P^_k over the first 16 columns of S_k
      } else {
        tmem_st32(ts, pk);  // P_k over the first 32 columns of S_k
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[sb]);
    }
    // ---------------- linear branch operand: phi~(q_r) in place of q_r
    float esum = 0.f, edotz = 0.f;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, a.err, DEV_TIMEOUT_TMA));
    if (ok && U >= 1)  // every S MMA has read Q once the last score tile is done
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[(U - 1) & 1], ((U - 1) >> 1) & 1, a.err,
                                             DEV_TIMEOUT_MMA));
    if (ok) {
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(sQ + (c / 8) * 16384 + sw128_offset(r, (c % 8) * 16));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fmaxf(__low2float(p2[e]), __high2float(p2[e])));
      }
      const float nmx = -mx * LOG2E;
      // softmax over d: e = 2^((q - max q) log2 e), phi = e / sum(e);
      // elu + 1: e = phi itself, and the denominator's sum is 1
      const bool elu = a.phi == 1;
      auto feat = [&](float x) { return elu ? (x > 0.f ? x + 1.f : ex2(x * LOG2E)) : ex2(fmaf(x, LOG2E, nmx)); };
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        uint8_t* qp = sQ + (c / 8) * 16384 + sw128_offset(r, (c % 8) * 16);
        const uint4 v = *reinterpret_cast<const uint4*>(qp);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[e] = pack_bf16x2(feat(__low2float(p2[e])), feat(__high2float(p2[e])));
          const __nv_bfloat162 eb = *reinterpret_cast<const __nv_bfloat162*>(&o[e]);
          esum += __low2float(eb) + __high2float(eb);
        }
        *reinterpret_cast<uint4*>(qp) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      if (elu) esum = 1.f;
      fence_proxy_async_smem();
      mbar_arrive(phiq_ready);
      // phi~(q_r) . Z_i (Z arrives with this half's H tile)
      ok = __all_sync(0xffffffffu, mbar_wait(half == 1 && has_b ? hb_full : ha_full, 0, a.err,
                                             DEV_TIMEOUT_TMA));
      if (ok) {
        const uint8_t* zrow = sZ + (half == 1 && has_b ? L::CH * 128 : 0);
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(sQ + (c / 8) * 16384 + sw128_offset(r, (c % 8) * 16));
          const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&v);
          const uint4 zv = *reinterpret_cast<const uint4*>(zrow + (c / 8) * 128 + (c % 8) * 16);
          const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(&zv);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            edotz = fmaf(__low2float(e2[e]), __low2float(z2[e]),
                         fmaf(__high2float(e2[e]), __high2float(z2[e]), edotz));
        }
      }
    }
    // ---------------- epilogue
    if (ok && U >= 1)
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(U - 1) & 1], ((U - 1) >> 1) & 1, a.err,
                                             DEV_TIMEOUT_MMA));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(half == 0 ? la_full : lb_full, 0, a.err,
                                                   DEV_TIMEOUT_MMA));
    if (ok) {
      tc_fence_after();
      const int n = 64 * (half == 0 ? ia : ibl) + (r & 63);
      const bool store = (n < a.N) && (half == 0 || has_b);
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      // log-sum-exp of the row's scaled critical scores, for the backward:
      // sum_t exp(s_t) = 2^m * l with m in log2 units
      if (a.lse && store) a.lse[(int64_t)bh * a.N + n] = (m + log2f(l)) * 0.6931471805599453f;
      const float inv_den = 1.f / (edotz + esum * a.eps);
      float wa, wl;
      if (a.combine == 1) {
        const float al = a.alpha[bh];
        wa = al * inv_l;
        wl = (1.f - al) * inv_den;
      } else {
        wa = inv_l;
        wl = inv_den;
      }
      __nv_bfloat16* orow = a.O + (int64_t)b * a.so0 + (int64_t)h * a.so1 + (int64_t)n * a.so2;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32], lv[32];
        tmem_ld32(tl + COL_O + c0, ov);
        tmem_ld32(tl + COL_L + c0, lv);
        tmem_ld_wait();
        if (PV8) {  // dequantise P^ V^: s_V[c] / 448 with s_V = max|V[:, c]| / 448
#pragma unroll
          for (int c = 0; c < 32; ++c)
            ov[c] = __float_as_uint(__uint_as_float(ov[c]) *
                                    (__uint_as_float(a.vmax[(int64_t)bh * D + c0 + c]) * (1.f / 200704.f)));
        }
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = 8 * v + e;
              const float bias = (a.combine == 0 && a.proj_b) ? __ldg(a.proj_b + c0 + c) : 0.f;
              y[e] = __uint_as_float(ov[c]) * wa + __uint_as_float(lv[c]) * wl + bias;
            }
            dst[v] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                                pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
          }
          if (a.os) {  // the sparse branch's output in fp32, for the backward
            float4* od = reinterpret_cast<float4*>(a.os + ((int64_t)bh * a.N + n) * D + c0);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              od[v] = make_float4(__uint_as_float(ov[4 * v]) * inv_l, __uint_as_float(ov[4 * v + 1]) * inv_l,
                                  __uint_as_float(ov[4 * v + 2]) * inv_l, __uint_as_float(ov[4 * v + 3]) * inv_l);
          }
        }
      }
      if (half == 0) {  // L_a has been read: the S/P region can take L_b
        tc_fence_before();
        mbar_arrive(la_free);
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

template <int D, int QK8, bool PV8>
static cudaError_t launch_fused_t(const CUtensorMap& mapQ, const CUtensorMap& mapK,
                                  const CUtensorMap& mapV, const CUtensorMap& mapH,
                                  const CUtensorMap& mapZ, const CUtensorMap& mapQ8,
                                  const CUtensorMap& mapK8, const FusedArgs& a, int BH,
                                  cudaStream_t s) {
  const size_t smem = FusedSmem<D, (QK8 != 0)>::bytes(a.Tkv);
  cudaError_t e = cudaFuncSetAttribute(sla_fused_kernel<D, QK8, PV8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Tq + 1) / 2, BH);
  sla_fused_kernel<D, QK8, PV8><<<grid, 192, smem, s>>>(mapQ, mapK, mapV, mapH, mapZ, mapQ8, mapK8, a);
  return cudaGetLastError();
}

cudaError_t launch_fused(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                         const CUtensorMap& mapH, const CUtensorMap& mapZ, const CUtensorMap& mapQ8,
                         const CUtensorMap& mapK8, const FusedArgs& a, int D, int qk8, bool pv8, int BH,
                         cudaStream_t s) {
#define SLA_FUSED(d_, q_, p_) launch_fused_t<d_, q_, p_>(mapQ, mapK, mapV, mapH, mapZ, mapQ8, mapK8, a, BH, s)
  if (pv8) return qk8 == 2 ? SLA_FUSED(128, 2, true) : (qk8 == 1 ? SLA_FUSED(128, 1, true) : SLA_FUSED(128, 0, true));
  if (qk8 == 2) return SLA_FUSED(128, 2, false);
  if (qk8 == 1) return SLA_FUSED(128, 1, false);
  return D == 128 ? SLA_FUSED(128, 0, false) : SLA_FUSED(64, 0, false);
#undef SLA_FUSED
}

}  // namespace sla
