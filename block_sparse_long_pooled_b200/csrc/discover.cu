// Stage 1b: pattern discovery and compaction (FlashPrefill V2 paper page: the abstract's
// "max-based dynamic thresholding", Table 9's parameter alpha, Table 7's "CSR of selected
// blocks, per KV head"; backend flags of the nestfrontier.com write-up: sink, window,
// last-n-blocks, min sparse q len).
//
// discover_kernel: one CTA per (sequence, tile of TI query blocks, KV head).  The G pooled
//   queries of every query block in the tile and 32-block chunks of pooled keys are staged
//   in shared memory; each thread forms 4 fp32 dot products per chunk.  All scores of the
//   tile stay in shared memory, so the row max and the threshold test need no second
//   pass.  Output: one bit per causal (row, key block) plus a kept count per row.
// scan_kernel: exclusive scan of the row counts into row_ptr (one CTA).
// scatter_kernel: one warp per row turns its bit words into ascending column ids.
#include <math_constants.h>

#include "fp2_device.cuh"
#include "fp2_kernels.h"

namespace fp2 {

constexpr int kJC = 32;  // key blocks per staged chunk

FP2_DEVICE void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
FP2_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FP2_DEVICE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(256) discover_kernel(const DiscArgs a, const Fp2Plan P) {
  extern __shared__ __align__(16) float smem[];
  int r, it, g;
  if (!map_heavy_first(P, a.TI, a.Hkv, blockIdx.x, r, it, g)) return;
  // Query block i of the sequence (or chunk) is absolute key block I = pre + i.
  const int N = P.nblk[r], L = P.len[r], pre = P.pre_blk[r];
  const int G = a.G;
  const int i0 = it * a.TI, i1 = min(N, i0 + a.TI);
  const int nI = i1 - i0, rows = nI * G;
  const int bo = P.blk_off[r], kbo = P.k_blk_off[r];
  const int J1 = pre + i1;  // key blocks [0, J1) are visible to some row of the tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool dense = a.dense_all || L < a.min_sparse_len;

  if (dense) {  // every causal block kept
    for (int ii = warp; ii < nI; ii += 8) {
      const int i = i0 + ii, I = pre + i;
      const int64_t row = static_cast<int64_t>(bo + i) * a.Hkv + g;
      const int nw = (I + 32) / 32;
      for (int w = lane; w < nw; w += 32) {
        const int nbits = min(32, I + 1 - 32 * w);
        a.bitmask[row * a.W + w] = nbits == 32 ? 0xFFFFFFFFu : ((1u << nbits) - 1u);
      }
      if (lane == 0) a.counts[row] = I + 1;
    }
    return;
  }

  constexpr int KS = D + 4;  // padded pooled-key row (conflict-free float4 reads)
  float* qs = smem;                       // [TI*G][D]
  float* ks = qs + a.TI * G * D;          // [2][kJC][KS]: chunk being used, chunk in flight
  float* sc = ks + 2 * kJC * KS;          // [TI*G][SP]
  float* thr = sc + a.TI * G * a.SP;      // [TI*G]

  for (int idx = tid; idx < rows * (D / 4); idx += 256) {
    const int row = idx / (D / 4), c4 = idx % (D / 4);
    const int ii = row / G, hl = row % G;
    reinterpret_cast<float4*>(qs)[row * (D / 4) + c4] = reinterpret_cast<const float4*>(
        a.qbar)[(static_cast<int64_t>(bo + i0 + ii) * a.Hq + g * G + hl) * (D / 4) + c4];
  }

  // Key chunks are double-buffered with cp.async: chunk c+1 streams in while chunk c is used.
  auto load_chunk = [&](int j0, int buf) {
    float* kb = ks + buf * (kJC * KS);
    for (int idx = tid; idx < kJC * (D / 4); idx += 256) {
      const int jj = idx / (D / 4), c4 = idx % (D / 4);
      const int j = j0 + jj;
      float* dst = &kb[jj * KS + c4 * 4];
      if (j < J1)
        cp_async16(dst, &a.kbar[(static_cast<int64_t>(kbo + j) * a.Hkv + g) * D + c4 * 4]);
      else
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_commit();
  };
  load_chunk(0, 0);
  for (int j0 = 0, it = 0; j0 < J1; j0 += kJC, ++it) {
    const int buf = it & 1;
    if (j0 + kJC < J1) {
      load_chunk(j0 + kJC, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // chunk `buf` (and, on the first pass, the query rows) visible to all
    const float* kb = ks + buf * (kJC * KS);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(&kb[lane * KS + k]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int row = warp + 8 * u;
        if (row < rows) {
          const float4 qv = *reinterpret_cast<const float4*>(&qs[row * D + k]);
          acc[u] = fmaf(qv.x, kv.x, acc[u]);
          acc[u] = fmaf(qv.y, kv.y, acc[u]);
          acc[u] = fmaf(qv.z, kv.z, acc[u]);
          acc[u] = fmaf(qv.w, kv.w, acc[u]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int row = warp + 8 * u;
      if (row < rows && j0 + lane < J1) sc[row * a.SP + j0 + lane] = acc[u] * a.scale;
    }
    __syncthreads();  // every thread is done with chunk `buf` before it is refilled
  }
  __syncthreads();

  // Row max over every causal key block (forced ones included), then the threshold.
  for (int row = warp; row < rows; row += 8) {
    const int I = pre + i0 + row / G;
    float m = -CUDART_INF_F;
    for (int j = lane; j <= I; j += 32) m = fmaxf(m, sc[row * a.SP + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) thr[row] = m + a.ln_alpha;
  }
  __syncthreads();

  const int win = max(a.window, 1);
  for (int ii = warp; ii < nI; ii += 8) {
    const int i = i0 + ii, I = pre + i;
    const int64_t row_id = static_cast<int64_t>(bo + i) * a.Hkv + g;
    const int nw = (I + 32) / 32;
    const bool last_rows = i >= N - a.last_n;
    int cnt = 0;
    for (int w = 0; w < nw; ++w) {
      const int j = w * 32 + lane;
      bool keep = false;
      if (j <= I) {
        keep = last_rows || (j < a.sink) || (j > I - win);
        for (int hl = 0; hl < G && !keep; ++hl) keep = sc[(ii * G + hl) * a.SP + j] >= thr[ii * G + hl];
      }
      const uint32_t bits = __ballot_sync(0xFFFFFFFFu, keep);
      if (lane == 0) a.bitmask[row_id * a.W + w] = bits;
      cnt += __popc(bits);
    }
    if (lane == 0) a.counts[row_id] = cnt;
  }
}

__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ counts, int64_t rows,
                                                    int32_t* __restrict__ row_ptr, int64_t capacity,
                                                    uint32_t* status) {
  __shared__ long long wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t seg = (rows + 1023) / 1024;
  const int64_t s0 = min(rows, tid * seg), s1 = min(rows, s0 + seg);
  long long local = 0;
  for (int64_t x = s0; x < s1; ++x) local += counts[x];
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;  // inclusive per warp
  }
  __syncthreads();
  long long run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
  for (int64_t x = s0; x < s1; ++x) {
    row_ptr[x] = static_cast<int32_t>(run);
    run += counts[x];
  }
  if (tid == 0) {
    const long long total = wsum[31];
    row_ptr[rows] = static_cast<int32_t>(total);
    if (total > capacity) set_status(status, FP2_DEV_CAPACITY);
  }
}

__global__ void __launch_bounds__(256) scatter_kernel(const uint32_t* __restrict__ bitmask, int W,
                                                      const int32_t* __restrict__ row_ptr,
                                                      int32_t* __restrict__ col_idx, int64_t capacity, int Hkv,
                                                      int64_t rows, const Fp2Plan P) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int b = static_cast<int>(row / Hkv);
  const int r = seq_of_block(P, b);
  const int I = P.pre_blk[r] + (b - P.blk_off[r]);  // absolute key block of the row's query block
  const int nw = (I + 32) / 32;
  const int base = row_ptr[row];
  if (row_ptr[row + 1] > capacity) return;
  int prefix = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bits = w < nw ? bitmask[row * W + w] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + prefix + incl - c;
    while (bits) {
      const int bp = __ffs(bits) - 1;
      bits &= bits - 1;
      col_idx[pos++] = w * 32 + bp;
    }
    prefix += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
}

size_t discover_smem_bytes(int D, int G, int TI, int SP) {
  return sizeof(float) * (static_cast<size_t>(TI) * G * D + 2 * kJC * (D + 4) + static_cast<size_t>(TI) * G * SP +
                          static_cast<size_t>(TI) * G);
}

cudaError_t launch_discover(const DiscArgs& a, const Fp2Plan& P, int64_t items, int64_t rows, int32_t* row_ptr,
                            int32_t* col_idx, int64_t capacity, cudaStream_t stream) {
  const size_t smem = discover_smem_bytes(a.D, a.G, a.TI, a.SP);
  cudaError_t e;
  if (a.D == 64) {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<64>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    discover_kernel<64><<<static_cast<unsigned>(items), 256, smem, stream>>>(a, P);
  } else {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<128>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    discover_kernel<128><<<static_cast<unsigned>(items), 256, smem, stream>>>(a, P);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scan_kernel<<<1, 1024, 0, stream>>>(a.counts, rows, row_ptr, capacity, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scatter_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(a.bitmask, a.W, row_ptr, col_idx, capacity,
                                                                           a.Hkv, rows, P);
  return cudaGetLastError();
}

}  // namespace fp2
