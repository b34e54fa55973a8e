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
// pairing_kernel: one CTA per head.  Overlap |C_i & C_c| of every block i with
// every candidate c = i + offset (sorted lists, merge count), then rounds of
// mutual best choice among unmatched blocks (ties: the smaller offset index),
// then the leftovers in index order.  Output pairs[bh][p] = (a, b), b = -1 for
// a single block; ceil(T / 2) pairs per head.  Lists: either fixed-length rows
// (lists + (bh T + i) len, ptr == nullptr) or CSR (lists + bh * stride, row i in
// [ptr[bh (T + 1) + i], ptr[bh (T + 1) + i + 1])), ascending in both.
#include "kernels.cuh"

namespace sla {

namespace {
constexpr int NCAND = 16;
__constant__ int kOffsets[NCAND] = {-1, 1, -2, 2, -23, 23, -24, 24, -25, 25, -26, 26, -48, 48, -49, 49};
constexpr int ROUNDS = 8;
}  // namespace

__global__ void __launch_bounds__(1024) pairing_kernel(const int32_t* __restrict__ lists,
                                                       const int32_t* __restrict__ ptr, int64_t stride, int Tq,
                                                       int len, int2* __restrict__ pairs) {
  extern __shared__ uint8_t psm[];
  uint16_t* ov = reinterpret_cast<uint16_t*>(psm);                 // [Tq][NCAND] overlaps
  int16_t* best = reinterpret_cast<int16_t*>(psm + 2 * (size_t)Tq * NCAND);  // [Tq]
  int16_t* mate = best + ((Tq + 7) & ~7);                          // [Tq], -1 = unmatched
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int32_t* L = ptr ? lists + (int64_t)bh * stride : lists + (int64_t)bh * Tq * len;
  const int32_t* P = ptr ? ptr + (int64_t)bh * (Tq + 1) : nullptr;
  for (int e = tid; e < Tq * NCAND; e += blockDim.x) {
    const int i = e / NCAND, c = i + kOffsets[e % NCAND];
    int cnt = 0;
    if (c >= 0 && c < Tq) {
      const int32_t* x = P ? L + P[i] : L + (int64_t)i * len;
      const int32_t* y = P ? L + P[c] : L + (int64_t)c * len;
      const int nx = P ? P[i + 1] - P[i] : len, ny = P ? P[c + 1] - P[c] : len;
      int u = 0, v = 0;
      while (u < nx && v < ny) {  // both rows ascending
        const int32_t a = x[u], b = y[v];
        cnt += a == b;
        u += a <= b;
        v += b <= a;
      }
    }
    ov[e] = (uint16_t)min(cnt, 65535);
  }
  for (int i = tid; i < Tq; i += blockDim.x) mate[i] = -1;
  __syncthreads();
  for (int round = 0; round < ROUNDS; ++round) {
    for (int i = tid; i < Tq; i += blockDim.x) {
      int bj = -1, bv = -1;
      if (mate[i] < 0) {
        for (int k = 0; k < NCAND; ++k) {
          const int c = i + kOffsets[k];
          if (c >= 0 && c < Tq && mate[c] < 0 && (int)ov[i * NCAND + k] > bv) {
            bv = ov[i * NCAND + k];
            bj = c;
          }
        }
      }
      best[i] = (int16_t)bj;
    }
    __syncthreads();
    for (int i = tid; i < Tq; i += blockDim.x) {
      const int j = best[i];
      if (j >= 0 && best[j] == i) mate[i] = (int16_t)j;  // mutual: both sides set their own entry
    }
    __syncthreads();
  }
  if (tid == 0) {
    int np = 0, pending = -1;
    int2* out = pairs + (int64_t)bh * ((Tq + 1) / 2);
    for (int i = 0; i < Tq; ++i) {
      const int j = mate[i];
      if (j >= 0) {
        if (i < j) out[np++] = make_int2(i, j);
      } else if (pending < 0) {
        pending = i;
      } else {
        out[np++] = make_int2(pending, i);
        pending = -1;
      }
    }
    if (pending >= 0) out[np++] = make_int2(pending, -1);
  }
}

size_t pairing_smem(int Tq) {
  return 2 * (size_t)Tq * NCAND + 2 * 2 * (size_t)((Tq + 7) & ~7);
}

static cudaError_t launch(const int32_t* lists, const int32_t* ptr, int64_t stride, int BH, int T, int len,
                          int2* pairs, cudaStream_t s) {
  const size_t smem = pairing_smem(T);
  cudaError_t e = cudaFuncSetAttribute(pairing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pairing_kernel<<<BH, 1024, smem, s>>>(lists, ptr, stride, T, len, pairs);
  return cudaGetLastError();
}

cudaError_t launch_pairing(const int32_t* lut, int BH, int Tq, int nh, int2* pairs, cudaStream_t s) {
  return launch(lut, nullptr, 0, BH, Tq, nh, pairs, s);
}

cudaError_t launch_pairing_csr(const int32_t* rows, const int32_t* ptr, int64_t stride, int BH, int T,
                               int2* pairs, cudaStream_t s) {
  return launch(rows, ptr, stride, BH, T, 0, pairs, s);
}

}  // namespace sla
