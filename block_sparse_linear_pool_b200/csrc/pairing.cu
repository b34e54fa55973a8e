// Which two blocks share a CTA of the fused forward and of the sparse backward.
//
// A CTA of 128 rows walks the union of its two blocks' lists: for two query
// blocks their critical lists (forward, dQ), for two key blocks the query blocks
// that have them critical (dK / dV).  The closer the two lists, the fewer union
// entries (tiles loaded, score tiles computed, hand-offs).  Adjacent blocks in
// token order (2p, 2p+1) share about 45% of their critical blocks on the video
// workloads; pairing each block with the most similar of its nearby blocks (same
// row, the previous / next grid row of a frame, the previous / next frame) cuts
// the union by 8-9%.  The result is the same for any pairing: a block outside
// one row's list contributes exact zeros to it.
//
// Two kernels per call:
//   pair_overlap_kernel  CTA = 64 blocks of one head: the lists of those blocks
//                        and of their candidates as bitsets in shared memory,
//                        then ov[i][k] = |C_i & C_{i + offset_k}| by popcount
//   pair_match_kernel    CTA = one head: rounds of mutual best choice among
//                        unmatched blocks (ties: the smaller offset index), the
//                        leftovers paired in index order; pairs written in the
//                        order of their first block (two block-wide scans)
// Output pairs[bh][p] = (a, b), b = -1 for a single block; ceil(T / 2) pairs per
// head.  Lists: either fixed-length rows (lists + (bh T + i) len, ptr == nullptr)
// or CSR (lists + bh * stride, row i in [ptr[bh (T + 1) + i], ptr[bh (T + 1) + i
// + 1])); entries are block indices in [0, ncol) (others are skipped: the
// kernels that follow report them).
#include "kernels.cuh"

namespace sla {

namespace {
constexpr int NCAND = 16;
constexpr int HALO = 49;  // largest |offset|
__constant__ int kOffsets[NCAND] = {-1, 1, -2, 2, -23, 23, -24, 24, -25, 25, -26, 26, -48, 48, -49, 49};
constexpr int ROUNDS = 8;
constexpr int RB = 64;        // blocks per overlap CTA
constexpr int OV_THREADS = 512;
constexpr int MATCH_THREADS = 1024;

// words per bitset row; odd, so that the rows that one warp reads at the same
// word index fall into different banks
__host__ __device__ inline int bits_stride(int ncol) { return ((ncol + 31) >> 5) | 1; }

// exclusive scan of one int per thread over the block; *total = the sum
__device__ int block_exclusive_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const int pre = (warp > 0 ? wsum[warp - 1] : 0) + x - v;
  *total = wsum[nw - 1];
  __syncthreads();  // wsum is reused by the next scan
  return pre;
}
}  // namespace

__global__ void __launch_bounds__(OV_THREADS) pair_overlap_kernel(const int32_t* __restrict__ lists,
                                                                  const int32_t* __restrict__ ptr,
                                                                  int64_t stride, int T, int len, int ncol,
                                                                  uint16_t* __restrict__ ov) {
  extern __shared__ uint32_t pbits[];  // [hi - lo][WS] bitsets of blocks lo .. hi-1
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, i0 = blockIdx.x * RB;
  const int W = (ncol + 31) >> 5, WS = bits_stride(ncol);
  const int lo = max(0, i0 - HALO), hi = min(T, i0 + RB + HALO);
  for (int x = tid; x < (hi - lo) * WS; x += blockDim.x) pbits[x] = 0u;
  __syncthreads();
  const int32_t* L = ptr ? lists + (int64_t)bh * stride : lists + (int64_t)bh * T * len;
  const int32_t* P = ptr ? ptr + (int64_t)bh * (T + 1) : nullptr;
  for (int r = lo + warp; r < hi; r += blockDim.x >> 5) {  // one warp per list
    const int32_t* row = P ? L + P[r] : L + (int64_t)r * len;
    const int n = P ? P[r + 1] - P[r] : len;
    uint32_t* br = pbits + (r - lo) * WS;
    for (int e = lane; e < n; e += 32) {
      const int j = row[e];
      if (j >= 0 && j < ncol) atomicOr(&br[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  for (int t = tid; t < RB * NCAND; t += blockDim.x) {
    const int i = i0 + t / NCAND, k = t % NCAND, c = i + kOffsets[k];
    if (i >= T) continue;
    int cnt = 0;
    if (c >= 0 && c < T) {  // c in [lo, hi)
      const uint32_t* a = pbits + (i - lo) * WS;
      const uint32_t* b = pbits + (c - lo) * WS;
      for (int w = 0; w < W; ++w) cnt += __popc(a[w] & b[w]);
    }
    ov[((int64_t)bh * T + i) * NCAND + k] = (uint16_t)min(cnt, 65535);
  }
}

__global__ void __launch_bounds__(MATCH_THREADS) pair_match_kernel(const uint16_t* __restrict__ ovg, int T,
                                                                   int2* __restrict__ pairs) {
  extern __shared__ uint8_t psm[];
  uint16_t* ov = reinterpret_cast<uint16_t*>(psm);                            // [T][NCAND]
  int16_t* best = reinterpret_cast<int16_t*>(psm + 2 * (size_t)T * NCAND);   // [T]
  int16_t* mate = best + ((T + 7) & ~7);                                      // [T], -1 = unmatched
  int16_t* ulist = mate + ((T + 7) & ~7);                                     // [T] unmatched, by rank
  __shared__ int wsum[32];
  const int bh = blockIdx.x, tid = threadIdx.x;
  {
    const uint4* src = reinterpret_cast<const uint4*>(ovg + (int64_t)bh * T * NCAND);  // 32 B per block
    uint4* dst = reinterpret_cast<uint4*>(ov);
    for (int x = tid; x < 2 * T; x += blockDim.x) dst[x] = src[x];
  }
  for (int i = tid; i < T; i += blockDim.x) mate[i] = -1;
  __syncthreads();
  for (int round = 0; round < ROUNDS; ++round) {
    for (int i = tid; i < T; i += blockDim.x) {
      int bj = -1, bv = -1;
      if (mate[i] < 0) {
        for (int k = 0; k < NCAND; ++k) {
          const int c = i + kOffsets[k];
          if (c >= 0 && c < T && mate[c] < 0 && (int)ov[i * NCAND + k] > bv) {
            bv = ov[i * NCAND + k];
            bj = c;
          }
        }
      }
      best[i] = (int16_t)bj;
    }
    __syncthreads();
    for (int i = tid; i < T; i += blockDim.x) {
      const int j = best[i];
      if (j >= 0 && best[j] == i) mate[i] = (int16_t)j;  // mutual: both sides set their own entry
    }
    __syncthreads();
  }
  // each thread owns the contiguous blocks [c0, c1)
  const int chunk = (T + blockDim.x - 1) / blockDim.x;
  const int c0 = min(T, tid * chunk), c1 = min(T, c0 + chunk);
  int nu = 0;
  for (int i = c0; i < c1; ++i) nu += mate[i] < 0;
  int U;
  const int rank0 = block_exclusive_scan(nu, wsum, &U);  // unmatched blocks before c0
  {
    int r = rank0;
    for (int i = c0; i < c1; ++i)
      if (mate[i] < 0) ulist[r++] = (int16_t)i;
  }
  // a pair starts at a matched block whose mate is later, or at an unmatched
  // block of even rank (its partner: the unmatched block of the next rank)
  int ns = 0;
  {
    int r = rank0;
    for (int i = c0; i < c1; ++i) {
      const int m = mate[i];
      if (m < 0) ns += (r++ & 1) == 0;
      else ns += m > i;
    }
  }
  int total;
  int pos = block_exclusive_scan(ns, wsum, &total);  // also orders the ulist writes before the reads
  int2* out = pairs + (int64_t)bh * ((T + 1) / 2);
  int r = rank0;
  for (int i = c0; i < c1; ++i) {
    const int m = mate[i];
    if (m < 0) {
      if ((r & 1) == 0) out[pos++] = make_int2(i, r + 1 < U ? (int)ulist[r + 1] : -1);
      ++r;
    } else if (m > i) {
      out[pos++] = make_int2(i, m);
    }
  }
}

size_t pairing_overlap_bytes(int BH, int T) { return (size_t)BH * T * NCAND * 2; }

static cudaError_t launch(const int32_t* lists, const int32_t* ptr, int64_t stride, int BH, int T, int len,
                          int ncol, uint16_t* ov, int2* pairs, cudaStream_t s) {
  const size_t smem_ov = (size_t)(RB + 2 * HALO) * bits_stride(ncol) * 4;
  cudaError_t e = cudaFuncSetAttribute(pair_overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_ov);
  if (e != cudaSuccess) return e;
  pair_overlap_kernel<<<dim3((T + RB - 1) / RB, BH), OV_THREADS, smem_ov, s>>>(lists, ptr, stride, T, len,
                                                                               ncol, ov);
  const size_t smem_m = 2 * (size_t)T * NCAND + 3 * 2 * (size_t)((T + 7) & ~7);
  e = cudaFuncSetAttribute(pair_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_m);
  if (e != cudaSuccess) return e;
  pair_match_kernel<<<BH, MATCH_THREADS, smem_m, s>>>(ov, T, pairs);
  return cudaGetLastError();
}

cudaError_t launch_pairing(const int32_t* lut, int BH, int Tq, int nh, int ncol, uint16_t* ov, int2* pairs,
                           cudaStream_t s) {
  return launch(lut, nullptr, 0, BH, Tq, nh, ncol, ov, pairs, s);
}

cudaError_t launch_pairing_csr(const int32_t* rows, const int32_t* ptr, int64_t stride, int BH, int T,
                               int ncol, uint16_t* ov, int2* pairs, cudaStream_t s) {
  return launch(rows, ptr, stride, BH, T, 0, ncol, ov, pairs, s);
}

}  // namespace sla
