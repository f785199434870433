// Stage 1a: block-mean pooling of Q, K and V (FlashPrefill V2 paper page, Figure 3:
// Stage 1 "pools block-mean statistics"; ResearchPod episode: a block is scored from a
// simple average of its tokens).
//
// One pass over Q, K and V.  A CTA owns one pooled block b (B consecutive tokens of one
// sequence) and a 128-vector slice of the concatenated token row [Q row | K row | V row];
// each thread owns one 16-byte column vector of that row and walks the block's tokens
// with eight independent 16-byte streaming loads in flight, accumulating in fp32.  Paged
// K/V rows are gathered through the page table, whose entries for the block are read once per
// CTA.  HBM-bound: the only traffic is one read of Q, K, V and a (1/B)-sized write of the means.
#include "fp2_device.cuh"
#include "fp2_kernels.h"

namespace fp2 {

template <int DT>
struct Elt;
template <>
struct Elt<0> {  // f32
  static constexpr int kBytes = 4;
};
template <>
struct Elt<1> {  // bf16
  static constexpr int kBytes = 2;
};
template <>
struct Elt<2> {  // e4m3
  static constexpr int kBytes = 1;
};

FP2_DEVICE uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <int DT>
FP2_DEVICE void accumulate(const uint4& v, float* acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if constexpr (DT == 0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += __uint_as_float(w[e]);
  } else if constexpr (DT == 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((w[e] >> (16 * hlf)) & 0xFFFFu);
        const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
        acc[4 * e + 2 * hlf] += f.x;
        acc[4 * e + 2 * hlf + 1] += f.y;
      }
    }
  }
}

// One CTA per (key block b, slice of 128 vectors of the token row); block b is absolute block J
// of sequence r.  Its K and V rows are pooled into
// kbar/vbar row b (skipped for prefix blocks when they are already pooled); when J lies in the
// query chunk its Q rows are pooled into qbar row blk_off[r] + (J - pre_blk[r]).
template <int DT>
__global__ void __launch_bounds__(128) pool_kernel(const __grid_constant__ PoolArgs a,
                                                   const __grid_constant__ Fp2Plan P) {
  constexpr int VEC = 16 / Elt<DT>::kBytes;  // elements per 16-byte vector
  const int b = blockIdx.x;
  const int r = seq_of_key_block(P, b);
  const int J = b - P.k_blk_off[r];
  const int pre = P.pre_blk[r];
  const int Lk = pre * a.B + P.len[r];
  const int t0 = J * a.B;
  const int n = min(a.B, Lk - t0);
  const int VQ = a.Hq * a.D / VEC, VK = a.Hkv * a.D / VEC;
  const int vid = blockIdx.y * blockDim.x + threadIdx.x;
  // Paged K/V: the block's page ids (B / page_size of them, at most 8 since page_size >= 16, or
  // one page holding the whole block) are read from the page table once per CTA, so the token
  // loop below issues no dependent page-table loads.  Every thread reaches the barrier.
  __shared__ int pg_s[8];
  if (a.page_table != nullptr) {
    const int np = a.page_size >= a.B ? 1 : a.B / a.page_size;
    if (threadIdx.x < np) {
      const int tl = t0 + static_cast<int>(threadIdx.x) * a.page_size;
      int page = 0;
      if (tl < Lk) {
        page = a.page_table[static_cast<int64_t>(r) * a.max_pages + tl / a.page_size];
        if (page < 0 || page >= a.num_pages) {
          set_status(a.status, FP2_DEV_PAGE_OOB);
          page = 0;
        }
      }
      pg_s[threadIdx.x] = page;
    }
    __syncthreads();
  }
  if (vid >= VQ + 2 * VK || n <= 0) return;

  int which, col;
  if (vid < VQ) {
    which = 0;
    col = vid * VEC;
    if (J < pre) return;  // no query rows in prefix blocks
  } else if (vid < VQ + VK) {
    which = 1;
    col = (vid - VQ) * VEC;
  } else {
    which = 2;
    col = (vid - VQ - VK) * VEC;
  }
  if (which != 0 && a.kv_prefix_pooled && J < pre) return;
  const char* base = static_cast<const char*>(which == 0 ? a.q : (which == 1 ? a.k : a.v));
  const int64_t stride = which == 0 ? a.q_stride : a.kv_stride;
  const bool paged = (which != 0) && (a.page_table != nullptr);
  const int64_t tok_base = which == 0 ? static_cast<int64_t>(P.tok_off[r]) + (J - pre) * a.B
                                      : static_cast<int64_t>(P.k_tok_off[r]) + t0;
  const int out_row = which == 0 ? P.blk_off[r] + (J - pre) : b;

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;

  for (int t = 0; t < n; t += 8) {
    // Tokens t .. t+7 share one page (page_size >= 16 is a multiple of 8).
    int64_t row0 = tok_base + t;
    if (paged) {
      const int pslot = a.page_size >= a.B ? 0 : t / a.page_size;
      row0 = static_cast<int64_t>(pg_s[pslot]) * a.page_size + ((t0 + t) % a.page_size);
    }
    uint4 buf[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t + u < n) buf[u] = ld_stream_v4(base + ((row0 + u) * stride + col) * Elt<DT>::kBytes);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t + u < n) accumulate<DT>(buf[u], acc);
    if constexpr (DT == 2) {
      // E4M3: the V rows are also written as f16 (exact), in key-token order, for the f16 PV
      // product of the attention kernel.
      if (which == 2) {
        uint16_t* v16 = static_cast<uint16_t*>(a.v16);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (t + u < n) {
            const int64_t trow = static_cast<int64_t>(P.k_tok_off[r]) + t0 + t + u;
            const uint32_t w[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
            uint4 h0, h1;
            h0.x = e4m3x2_to_f16x2(w[0] & 0xFFFFu);
            h0.y = e4m3x2_to_f16x2(w[0] >> 16);
            h0.z = e4m3x2_to_f16x2(w[1] & 0xFFFFu);
            h0.w = e4m3x2_to_f16x2(w[1] >> 16);
            h1.x = e4m3x2_to_f16x2(w[2] & 0xFFFFu);
            h1.y = e4m3x2_to_f16x2(w[2] >> 16);
            h1.z = e4m3x2_to_f16x2(w[3] & 0xFFFFu);
            h1.w = e4m3x2_to_f16x2(w[3] >> 16);
            uint4* dst16 = reinterpret_cast<uint4*>(v16 + trow * a.Hkv * a.D + col);
            dst16[0] = h0;
            dst16[1] = h1;
          }
        }
      }
    }
  }

  const float descale = which == 0 ? a.q_descale : (which == 1 ? a.k_descale : a.v_descale);
  const float fn = static_cast<float>(n);
  float mean_raw[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) mean_raw[e] = acc[e] / fn;

  const int H = which == 0 ? a.Hq : a.Hkv;
  float* dst = which == 0 ? a.qbar : (which == 1 ? a.kbar : a.vbar);
  float4* d4 = reinterpret_cast<float4*>(dst + static_cast<int64_t>(out_row) * H * a.D + col);
#pragma unroll
  for (int e = 0; e < VEC / 4; ++e)
    d4[e] = make_float4(mean_raw[4 * e] * descale, mean_raw[4 * e + 1] * descale, mean_raw[4 * e + 2] * descale,
                        mean_raw[4 * e + 3] * descale);

  if (DT == 2 && which == 2) {
    // E4M3 vbar operand: f16 (the PV product runs in f16), stored-value domain.
    uint4 h[2];
    uint32_t* hw = reinterpret_cast<uint32_t*>(h);
#pragma unroll
    for (int e = 0; e < 8; ++e) hw[e] = pack_f16x2(mean_raw[2 * e], mean_raw[2 * e + 1]);
    uint4* d16 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.vbar_mma) + static_cast<int64_t>(out_row) * H * a.D + col);
    d16[0] = h[0];
    d16[1] = h[1];
  } else if (which != 0) {
    // Narrow copy in the MMA operand type (E4M3 stays in the stored, un-descaled domain).
    char* nb = static_cast<char*>(which == 1 ? a.kbar_mma : a.vbar_mma);
    uint4 out;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&out);
    if constexpr (DT == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) ow[e] = __float_as_uint(mean_raw[e]);
    } else if constexpr (DT == 1) {
#pragma unroll
      for (int e = 0; e < 4; ++e) ow[e] = pack_bf16x2(mean_raw[2 * e], mean_raw[2 * e + 1]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        ow[e] = pack_e4m3x4(mean_raw[4 * e], mean_raw[4 * e + 1], mean_raw[4 * e + 2], mean_raw[4 * e + 3]);
    }
    *reinterpret_cast<uint4*>(nb + (static_cast<int64_t>(out_row) * H * a.D + col) * Elt<DT>::kBytes) = out;
  }
}

cudaError_t launch_pool(int dtype, const PoolArgs& a, const Fp2Plan& P, cudaStream_t stream) {
  const int elt = dtype == FP2_F32 ? 4 : (dtype == FP2_BF16 ? 2 : 1);
  const int vec = 16 / elt;
  const int nvec = (a.Hq + 2 * a.Hkv) * a.D / vec;
  // 128 threads per CTA: the vector counts of the usual head layouts ((Hq + 2 Hkv) x d / vector)
  // are multiples of 128, so no CTA carries idle threads.
  dim3 grid(P.total_k_blocks, (nvec + 127) / 128);
  if (dtype == FP2_F32)
    pool_kernel<0><<<grid, 128, 0, stream>>>(a, P);
  else if (dtype == FP2_BF16)
    pool_kernel<1><<<grid, 128, 0, stream>>>(a, P);
  else
    pool_kernel<2><<<grid, 128, 0, stream>>>(a, P);
  return cudaGetLastError();
}

}  // namespace fp2
