// Stage 1b: pattern discovery and compaction (FlashPrefill V2 paper page: the abstract's
// "max-based dynamic thresholding", Table 9's parameter alpha, Table 7's "CSR of selected
// blocks, per KV head"; backend flags of the nestfrontier.com write-up: sink, window,
// last-n-blocks, min sparse q len).
//
// discover_kernel: one CTA (16 warps) per (sequence, tile of TI query blocks, KV head).  The G
//   pooled queries of every query block in the tile (up to 32 rows) and stages of 256 pooled
//   keys x 16 dimensions are staged in shared memory (cp.async, a ring of three buffers); the
//   scores are a small fp32 GEMM in which each thread owns 8 rows x 2 keys and each warp 8 rows
//   x 64 keys.  All scores of the tile stay in shared memory, so the row max and the threshold
//   test need no second pass.  Output: one bit per causal (row, key block) plus a kept count
//   per row.
// scan_kernel: exclusive scan of the row counts into row_ptr (one CTA).
// scatter_kernel: one warp per row turns its bit words into ascending column ids.
#include <math_constants.h>

#include "fp2_device.cuh"
#include "fp2_kernels.h"

namespace fp2 {

constexpr int kThreads = 512;  // 16 warps
constexpr int kWarps = kThreads / 32;
constexpr int kKC = 256;       // key blocks per staged chunk (4 key groups x 64)
constexpr int kDS = 16;        // head dimensions per stage
constexpr int kKS = kDS + 4;   // padded stage row (conflict-free 16-byte reads)
constexpr int kNB = 3;         // stage buffers: two stages in flight while one is used
constexpr int kRows = 32;      // score rows a CTA computes (TI * G <= 32; the rest are zero)

FP2_DEVICE void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
// 16-byte shared-memory load kept where it is written (volatile: not sunk towards its use).
FP2_DEVICE float4 lds128(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
FP2_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FP2_DEVICE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads) discover_kernel(const DiscArgs a, const Fp2Plan P) {
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
    for (int ii = warp; ii < nI; ii += kWarps) {
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

  constexpr int QS = D + 4;  // padded pooled-query row
  constexpr int NH = D / kDS;  // stages per key chunk
  const int SPP = a.SP + 8;    // score row stride
  float* qs = smem;                    // [kRows][QS]
  float* ks = qs + kRows * QS;         // [kNB][kKC][kKS]: stage being used, two in flight
  float* sc = ks + kNB * kKC * kKS;    // [TI*G][SPP]
  float* thr = sc + a.TI * G * SPP;    // [32]
  int* cnt = reinterpret_cast<int*>(thr + 32);  // [32] kept blocks per query block

  for (int idx = tid; idx < kRows * (D / 4); idx += kThreads) {
    const int row = idx / (D / 4), c4 = idx % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < rows) {
      const int ii = row / G, hl = row % G;
      v = reinterpret_cast<const float4*>(a.qbar)[(static_cast<int64_t>(bo + i0 + ii) * a.Hq + g * G + hl) * (D / 4) + c4];
    }
    *reinterpret_cast<float4*>(&qs[row * QS + c4 * 4]) = v;
  }
  if (tid < 32) cnt[tid] = 0;

  // Stage st covers key blocks [c*kKC, c*kKC + kKC) and dimensions [h*kDS, h*kDS + kDS) with
  // c = st / NH, h = st % NH; a ring of kNB buffers keeps stages st+1 and st+2 streaming in
  // while stage st is used (an L2 round trip is longer than one stage's arithmetic).
  // Each thread copies the same two 16-byte pieces of every stage: key rows jl and jl + 128 of
  // the chunk, dimensions [4*c4, 4*c4 + 4) of the stage.
  const int nst = (J1 + kKC - 1) / kKC * NH;
  const int jl = tid >> 2, c4l = tid & 3;
  const int64_t key_stride = static_cast<int64_t>(a.Hkv) * D;
  const float* kbase = a.kbar + (static_cast<int64_t>(kbo + jl) * a.Hkv + g) * D + c4l * 4;
  auto load_stage = [&](int st, int buf) {
    const int j0 = (st / NH) * kKC, d0 = (st % NH) * kDS;
    float* dst = ks + buf * (kKC * kKS) + jl * kKS + c4l * 4;
    const float* src = kbase + j0 * key_stride + d0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (j0 + jl + 128 * q < J1)
        cp_async16(dst + 128 * q * kKS, src + 128 * q * key_stride);
      else
        *reinterpret_cast<float4*>(dst + 128 * q * kKS) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_commit();
  };
  // Thread tile: rows 8 * (warp & 3) + n (n < 8) and keys 64 * (warp >> 2) + lane + 32m (m < 2)
  // of the chunk.  The query loads of a warp are pure broadcasts (one address) and its key
  // loads read 32 distinct rows, so every shared-memory wavefront carries 128 useful bytes.
  const int r0 = 8 * (warp & 3);
  const int kb0 = 64 * (warp >> 2) + lane;
  float acc[8][2];
#pragma unroll
  for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = 0.f;

  load_stage(0, 0);
  if (nst > 1) load_stage(1, 1);
  for (int st = 0; st < nst; ++st) {
    if (st + 1 < nst)
      cp_async_wait<1>();  // stage st has landed; stage st+1 may still be in flight
    else
      cp_async_wait<0>();
    // Stage st (and, on the first pass, the query rows) is visible to all; every thread is
    // done with stage st-1, whose buffer the next load refills.
    __syncthreads();
    if (st + 2 < nst) load_stage(st + 2, (st + 2) % kNB);
    const int h = st % NH, j0 = (st / NH) * kKC;
    if (j0 + 64 * (warp >> 2) < J1 && r0 < rows) {  // warps with no visible key or no row idle
      const uint32_t kp = smem_u32(ks + (st % kNB) * (kKC * kKS) + kb0 * kKS);
      const uint32_t qp = smem_u32(qs + r0 * QS + h * kDS);
      // Software pipeline: the operands of step k+1 are requested before the FMAs of step k, so
      // each warp's shared-memory loads overlap its own arithmetic (the warps of a CTA run in
      // lock step between barriers, so overlap across warps cannot be relied on).
      float4 qv[2][8], kv[2][2];
      auto load_step = [&](int k, int b) {
#pragma unroll
        for (int n = 0; n < 8; ++n) qv[b][n] = lds128(qp + 4u * (n * QS + k));
#pragma unroll
        for (int m = 0; m < 2; ++m) kv[b][m] = lds128(kp + 4u * (32 * m * kKS + k));
      };
      load_step(0, 0);
#pragma unroll
      for (int k = 0; k < kDS; k += 4) {
        const int b = (k >> 2) & 1;
        if (k + 4 < kDS) load_step(k + 4, b ^ 1);
        // Dimension by dimension over all 16 accumulators: consecutive FMAs are independent.
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m) acc[n][m] = fmaf(qv[b][n].x, kv[b][m].x, acc[n][m]);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m) acc[n][m] = fmaf(qv[b][n].y, kv[b][m].y, acc[n][m]);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m) acc[n][m] = fmaf(qv[b][n].z, kv[b][m].z, acc[n][m]);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m) acc[n][m] = fmaf(qv[b][n].w, kv[b][m].w, acc[n][m]);
      }
      if (h == NH - 1) {  // the chunk's dot products are complete
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int row = r0 + n, j = j0 + kb0 + 32 * m;
            if (row < rows && j < J1) sc[row * SPP + j] = acc[n][m] * a.scale;
            acc[n][m] = 0.f;
          }
      }
    }
  }
  __syncthreads();

  // Row max over every causal key block (forced ones included), then the threshold.  Four
  // independent running maxima per lane.
  for (int row = warp; row < rows; row += kWarps) {
    const int I = pre + i0 + row / G;
    const float* sr = sc + row * SPP;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, m2 = -CUDART_INF_F, m3 = -CUDART_INF_F;
    int j = lane;
    for (; j + 96 <= I; j += 128) {
      m0 = fmaxf(m0, sr[j]);
      m1 = fmaxf(m1, sr[j + 32]);
      m2 = fmaxf(m2, sr[j + 64]);
      m3 = fmaxf(m3, sr[j + 96]);
    }
    for (; j <= I; j += 32) m0 = fmaxf(m0, sr[j]);
    float m = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) thr[row] = m + a.ln_alpha;
  }
  __syncthreads();

  // One warp per (query block, 32-block word): forced blocks, or any head of the group at or
  // above its threshold.
  const int win = max(a.window, 1);
  const int wmax = (J1 - 1 + 32) / 32;  // words of the tile's last query block
  for (int p = warp; p < nI * wmax; p += kWarps) {
    const int ii = p / wmax, w = p % wmax;
    const int i = i0 + ii, I = pre + i;
    if (w >= (I + 32) / 32) continue;
    const int j = w * 32 + lane;
    bool keep = false;
    if (j <= I) {
      keep = (i >= N - a.last_n) || (j < a.sink) || (j > I - win);
      for (int hl = 0; hl < G; ++hl) keep |= sc[(ii * G + hl) * SPP + j] >= thr[ii * G + hl];
    }
    const uint32_t bits = __ballot_sync(0xFFFFFFFFu, keep);
    if (lane == 0) {
      a.bitmask[(static_cast<int64_t>(bo + i) * a.Hkv + g) * a.W + w] = bits;
      atomicAdd(&cnt[ii], __popc(bits));
    }
  }
  __syncthreads();
  if (tid < nI) a.counts[static_cast<int64_t>(bo + i0 + tid) * a.Hkv + g] = cnt[tid];
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
  return sizeof(float) * (static_cast<size_t>(kRows) * (D + 4) + kNB * kKC * kKS +
                          static_cast<size_t>(TI) * G * (SP + 8) + 64);
}

cudaError_t launch_discover(const DiscArgs& a, const Fp2Plan& P, int64_t items, int64_t rows, int32_t* row_ptr,
                            int32_t* col_idx, int64_t capacity, cudaStream_t stream) {
  const size_t smem = discover_smem_bytes(a.D, a.G, a.TI, a.SP);
  cudaError_t e;
  if (a.D == 64) {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<64>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    discover_kernel<64><<<static_cast<unsigned>(items), kThreads, smem, stream>>>(a, P);
  } else {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<128>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    discover_kernel<128><<<static_cast<unsigned>(items), kThreads, smem, stream>>>(a, P);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scan_kernel<<<1, 1024, 0, stream>>>(a.counts, rows, row_ptr, capacity, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scatter_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(a.bitmask, a.W, row_ptr, col_idx, capacity,
                                                                           a.Hkv, rows, P);
  return cudaGetLastError();
}

}  // namespace fp2
