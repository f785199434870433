// Stage 1b: pattern discovery and compaction (FlashPrefill V2 paper page: the abstract's
// "max-based dynamic thresholding", Table 9's parameter alpha, Table 7's "CSR of selected
// blocks, per KV head"; backend flags of the nestfrontier.com write-up: sink, window,
// last-n-blocks, min sparse q len).
//
// discover_kernel: one CTA per (sequence, tile of TI = 128 / G query blocks, KV head).  Its 128
//   score rows are the (query block, head) pairs of the tile (row m = query block m / G, head
//   m % G of the group) and form the M = 128 operand of tcgen05 MMAs; pooled keys stream in chunks
//   of 128 key blocks (N = 128) and the scores of a chunk land in tensor memory, one row per TMEM
//   lane.  The pooled means are fp32; the decision to keep a block must match an fp64 evaluation
//   outside a 1e-3 band, so each operand x is split into two bf16 planes, hi = bf16(x) and
//   lo = bf16(x - hi), and a score is hi.hi + hi.lo + lo.hi (three bf16 MMAs accumulating in
//   fp32): the dropped lo.lo term and the rounding of lo are both ~2^-16 of |x|, far inside the
//   band.  The rows need their maximum over every causal key block before any block can be
//   tested, so the chunks run twice: pass 1 takes the row maxima, pass 2 recomputes the scores
//   (the tensor cores are cheap next to everything else here) and tests them against
//   max + ln alpha.  Warp roles (416 threads):
//     warps 0-3   epilogue: one TMEM lane quarter each, so thread t owns score row t; reads a
//                 chunk's 128 scores, releases the TMEM buffer, pass 1 updates the row max, pass
//                 2 builds 4 words of kept bits that are OR-ed over the G heads of each query
//                 block in shared memory (GQA union), and writes the words (with the forced
//                 blocks: sink, window/diagonal, last-n rows) and the per-row counts.
//     warps 4-11  converters: load fp32 pooled rows (coalesced 16-byte loads, 16 in flight per
//                 thread), split them into the hi/lo bf16 planes and store them in the
//                 128-byte-swizzled K-major layout the MMA reads: the query tile once, then
//                 every key chunk of both passes into a ring of NST stages.
//     warp 12     MMA issuer: 3 x D/16 MMAs per chunk into one of four 128-column TMEM buffers.
//   Every wait is an mbarrier wait with a time limit; after a timeout every role runs its loop to
//   the end without work, so the index written is still consistent (forced blocks only) and the
//   status word says FP2_DEV_TIMEOUT.
// scan_kernel: exclusive scan of the row counts into row_ptr (one CTA).
// scatter_kernel: one warp per row turns its bit words into ascending column ids.
#include <math_constants.h>

#include "fp2_device.cuh"
#include "fp2_kernels.h"

namespace fp2 {

template <int D>
struct DiscCfg {
  static constexpr int ROWS = 128;                 // M: score rows of a CTA
  static constexpr int KEYS = 128;                 // N: key blocks per chunk
  static constexpr int UPR = D / 8;                // 8-element units per pooled row
  static constexpr int PLANE = 128 * D * 2;        // one bf16 plane of 128 rows (query tile or key chunk)
  static constexpr int NST = D == 64 ? 4 : 2;      // key-chunk stages (hi + lo planes each)
  static constexpr int NBUF = 4;                   // 128-column score buffers in TMEM
  static constexpr int NCONV = 8;                  // converter warps
  static constexpr int THREADS = (4 + NCONV + 1) * 32;
  static constexpr int OFF_AHI = 0, OFF_ALO = PLANE, OFF_B = 2 * PLANE;
  static constexpr int OFF_BAR = OFF_B + NST * 2 * PLANE;
  static constexpr int NBAR = 1 + 2 * NST + 2 * NBUF + 1;
  static constexpr int OFF_UNION = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;  // [2][128][4] u32
  static constexpr int OFF_CNT = OFF_UNION + 2 * 128 * 4 * 4;            // [128] int
  static constexpr int OFF_MISC = OFF_CNT + 128 * 4;                     // TMEM address, abort flag
  static constexpr int OFF_CHK = OFF_MISC + 16;                          // checked builds: 16 counters
  static constexpr int SMEM_BYTES = OFF_CHK + 64 + 1024;                 // + 1024-byte alignment slack
  // bf16 x bf16 -> f32, both operands K-major, M = 128, N = 128.
  static constexpr uint32_t IDESC = make_idesc(1u, 1u, 0u, 0u, 128u, 128u);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_BAR % 8 == 0 && OFF_UNION % 16 == 0 && OFF_CHK % 16 == 0 && NST <= 4 && NBUF <= 4,
                "shared-memory layout");
  static_assert((128 * UPR) % (NCONV * 32) == 0, "converter work split");
};

// 64 consecutive TMEM columns of this thread's lane, with the wait in the same statement so that
// no use of the registers is scheduled before the data has landed.
FP2_DEVICE void tmem_ld_row64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr + 0u), "r"(taddr + 32u)
      : "memory");
}

// Bounded wait used only to drain the MMAs in flight before TMEM is freed (ignores the abort flag).
FP2_DEVICE void drain_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) {
      set_status(status, FP2_DEV_TIMEOUT);
      return;
    }
  }
}

FP2_DEVICE void epilogue_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Bits of word w (blocks 32w .. 32w+31) that lie in [lo, hi].
FP2_DEVICE uint32_t range_bits(int lo, int hi, int w) {
  const int base = 32 * w;
  const int a = max(lo, base), b = min(hi, base + 31);
  if (a > b) return 0u;
  const int len = b - a + 1;
  return (len == 32 ? 0xFFFFFFFFu : ((1u << len) - 1u)) << (a - base);
}

// Split 8 fp32 values into the 16-byte hi and lo bf16 units: hi = bf16(x), lo = bf16(x - hi).
FP2_DEVICE void split_bf16x8(const float4& a, const float4& b, uint4& hi, uint4& lo) {
  const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    h[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
    const float r0 = x[2 * e] - __uint_as_float(h[e] << 16);
    const float r1 = x[2 * e + 1] - __uint_as_float(h[e] & 0xFFFF0000u);
    l[e] = pack_bf16x2(r0, r1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int D>
__global__ void __launch_bounds__(DiscCfg<D>::THREADS, 1) discover_kernel(const __grid_constant__ DiscArgs a,
                                                                         const __grid_constant__ Fp2Plan P) {
  using C = DiscCfg<D>;
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

  if (a.dense_all || L < a.min_sparse_len) {  // every causal block kept
    for (int ii = warp; ii < nI; ii += C::THREADS / 32) {
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

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* b_full = a_full + 1;
  uint64_t* b_empty = b_full + C::NST;
  uint64_t* s_full = b_empty + C::NST;
  uint64_t* s_empty = s_full + C::NBUF;
  uint64_t* mma_done = s_empty + C::NBUF;
  uint32_t* ubuf = reinterpret_cast<uint32_t*>(smem + C::OFF_UNION);  // [2][128][4]
  int* cnt = reinterpret_cast<int*>(smem + C::OFF_CNT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // Checked builds: hand-off counters, bumped by the signalling thread before its arrive or commit
  // and compared by the waiter with the exact count its own progress implies: chk[st] converter
  // fills of stage st (NCONV per use), chk[4 + st] releases of stage st by the MMA warp, chk[8 + b]
  // score chunks issued into TMEM buffer b, chk[12 + b] releases of buffer b (4 epilogue warps).
  volatile uint32_t* chk = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_CHK);
  auto bump = [&](int k) {
    if constexpr (FP2_CHECKED != 0) {
      atomicAdd(const_cast<uint32_t*>(chk + k), 1u);
      __threadfence_block();
    }
  };
  auto expect = [&](int k, int n) {
    if constexpr (FP2_CHECKED != 0) fp2_check(chk[k] == static_cast<uint32_t>(n), a.status);
  };

  const int nch = (J1 + C::KEYS - 1) / C::KEYS;
  const int nq = 2 * nch;  // pass 1 then pass 2 over the same chunks

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(a_full, C::NCONV);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&b_full[s], C::NCONV);
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    if constexpr (FP2_CHECKED != 0)
      for (int k = 0; k < 16; ++k) chk[k] = 0u;
    fence_mbar_init();
  }
  for (int x = tid; x < 2 * 128 * 4; x += C::THREADS) ubuf[x] = 0u;
  for (int x = tid; x < 128; x += C::THREADS) cnt[x] = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < 4 + C::NCONV) {
    // ------------------------------------------------------------------ converters
    // Thread ct owns the 8-element unit `col8` of rows r0, r0 + RSTEP, ...; unit col8 holds d
    // 8*col8 .. +7, which is 128-byte chunk col8 / 8, 16-byte unit col8 % 8 of the swizzled row.
    constexpr int RSTEP = C::NCONV * 32 / C::UPR;
    constexpr int NU = 128 / RSTEP;
    const int ct = tid - 128;
    const int col8 = ct % C::UPR, r0 = ct / C::UPR;
    const int chunk_off = (col8 >> 3) * (128 * 128);
    float4 x[NU][2];
    // Loads of a tile's rows into registers (issued before waiting for the stage they go to, so
    // their latency overlaps the MMAs of the chunks before), then the split and swizzled stores.
    auto load = [&](auto src_of) {
#pragma unroll
      for (int k = 0; k < NU; ++k) {
        const float* p = src_of(r0 + RSTEP * k);
        if (p != nullptr) {
          x[k][0] = __ldg(reinterpret_cast<const float4*>(p + 8 * col8));
          x[k][1] = __ldg(reinterpret_cast<const float4*>(p + 8 * col8 + 4));
        } else {
          x[k][0] = x[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    auto store = [&](uint8_t* hi_base, uint8_t* lo_base) {
#pragma unroll
      for (int k = 0; k < NU; ++k) {
        const int row = r0 + RSTEP * k;
        uint4 hi, lo;
        split_bf16x8(x[k][0], x[k][1], hi, lo);
        const int off = chunk_off + row * 128 + (((col8 & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(hi_base + off) = hi;
        *reinterpret_cast<uint4*>(lo_base + off) = lo;
      }
      fence_proxy_async_smem();  // the tensor core reads the planes through the async proxy
      __syncwarp();
    };
    const int64_t qrow0 = static_cast<int64_t>(bo + i0) * a.Hq + static_cast<int64_t>(g) * G;
    load([&](int m) -> const float* {
      if (m >= rows) return nullptr;
      return a.qbar + (qrow0 + static_cast<int64_t>(m / G) * a.Hq + (m % G)) * D;
    });
    store(smem + C::OFF_AHI, smem + C::OFF_ALO);
    if (lane == 0) mbar_arrive(a_full);
    for (int q = 0; q < nq; ++q) {
      const int stage = q % C::NST, use = q / C::NST;
      const int j0 = (q % nch) * C::KEYS;
      load([&](int n) -> const float* {
        const int j = j0 + n;
        if (j >= J1) return nullptr;
        return a.kbar + (static_cast<int64_t>(kbo + j) * a.Hkv + g) * D;
      });
      if (use > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&b_empty[stage], (use - 1) & 1, abort_flag, a.status)))
        break;
      if (use > 0 && lane == 0) expect(4 + stage, use);  // the MMA warp released this use's stage
      uint8_t* hb = smem + C::OFF_B + stage * 2 * C::PLANE;
      store(hb, hb + C::PLANE);
      if (lane == 0) {
        bump(stage);
        mbar_arrive(&b_full[stage]);
      }
    }
  } else if (warp == 4 + C::NCONV) {
    // ------------------------------------------------------------------ MMA issuer
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(a_full, 0, abort_flag, a.status));
    for (int q = 0; q < nq && ok; ++q) {
      const int stage = q % C::NST, buf = q % C::NBUF;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&b_full[stage], (q / C::NST) & 1, abort_flag, a.status));
      if (ok && lane == 0) expect(stage, C::NCONV * (q / C::NST + 1));
      if (ok && q >= C::NBUF) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s_empty[buf], ((q / C::NBUF) - 1) & 1, abort_flag, a.status));
        if (ok && lane == 0) expect(12 + buf, 4 * (q / C::NBUF));
      }
      if (!ok) break;
      tc_fence_after();
      const uint32_t dcol = tmem + buf * C::KEYS;
      const uint32_t bbase = sbase + C::OFF_B + stage * 2 * C::PLANE;
#pragma unroll
      for (int t = 0; t < 3; ++t) {  // hi.hi, hi.lo, lo.hi
        const uint64_t ad0 = smem_desc_sw128(sbase + (t == 2 ? C::OFF_ALO : C::OFF_AHI), 16, 1024);
        const uint64_t bd0 = smem_desc_sw128(bbase + (t == 1 ? C::PLANE : 0), 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = static_cast<uint32_t>((k >> 2) * (128 * 128) + (k & 3) * 32);
          umma_ss_warp<1>(dcol, ad0 + (off >> 4), bd0 + (off >> 4), C::IDESC, (t > 0 || k > 0) ? 1u : 0u);
        }
      }
      if (lane == 0) {
        bump(4 + stage);
        bump(8 + buf);
      }
      __syncwarp();
      umma_commit_warp(&b_empty[stage]);
      umma_commit_warp(&s_full[buf]);
    }
    umma_commit_warp(mma_done);
    if (lane == 0) drain_wait(mma_done, 0, a.status);
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------------ epilogue
    const int m = warp * 32 + lane;  // score row = TMEM lane
    const bool valid = m < rows;
    const int ii = valid ? m / G : 0;
    const int I = pre + i0 + ii;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float scale = a.scale;
    const int win = max(a.window, 1);
    float mrun = -CUDART_INF_F, thr = CUDART_INF_F;
    bool ok = true;
    for (int q = 0; q < nq; ++q) {
      const int buf = q % C::NBUF, c = q % nch, j0 = c * C::KEYS;
      const bool pass2 = q >= nch;
      if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[buf], (q / C::NBUF) & 1, abort_flag, a.status));
      if (ok && lane == 0) expect(8 + buf, q / C::NBUF + 1);
      if (ok) tc_fence_after();
      if (pass2 && q == nch) thr = mrun + a.ln_alpha;
      const int lim = I - j0;  // columns e <= lim are causal for this row
      // The chunk's 128 scores in two halves of 64 columns (fewer live registers).
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t v[64];
        if (ok) tmem_ld_row64(tmem + lane_base + buf * C::KEYS + hf * 64, v);
        if (hf == 1) {  // the buffer has been read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            bump(12 + buf);
            mbar_arrive(&s_empty[buf]);
          }
        }
        if (!ok || !valid) continue;
        const int lh = lim - hf * 64;  // causal limit within this half
        if (!pass2) {
          if (lh >= 63) {
            float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
            for (int e = 0; e < 64; e += 8)
#pragma unroll
              for (int u = 0; u < 4; ++u)
                m4[u] = fmax3(m4[u], __uint_as_float(v[e + 2 * u]) * scale, __uint_as_float(v[e + 2 * u + 1]) * scale);
            mrun = fmax3(mrun, fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          } else {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e <= lh) mrun = fmaxf(mrun, __uint_as_float(v[e]) * scale);
          }
        } else {
#pragma unroll
          for (int wh = 0; wh < 2; ++wh) {
            uint32_t bits = 0u;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = 32 * wh + e;
              const bool keep = (__uint_as_float(v[col]) * scale >= thr) && (col <= lh);
              bits |= static_cast<uint32_t>(keep) << e;
            }
            if (bits != 0u) atomicOr(&ubuf[((c & 1) * 128 + ii) * 4 + 2 * hf + wh], bits);
          }
        }
      }
      if (pass2) {
        epilogue_bar_sync();
        // Union over the heads of each query block is complete: add the forced blocks and write.
        for (int x = m; x < a.TI * 4; x += 128) {
          const int iw = x >> 2, wq = x & 3;
          const int i = i0 + iw;
          uint32_t* slot = &ubuf[((c & 1) * 128 + iw) * 4 + wq];
          if (i < i1) {
            const int Iw = pre + i, w = 4 * c + wq;
            if (w <= (Iw >> 5)) {
              uint32_t word = *slot;
              word |= range_bits(0, a.sink - 1, w) | range_bits(Iw - win + 1, Iw, w);
              if (i >= N - a.last_n) word = 0xFFFFFFFFu;
              word &= range_bits(0, Iw, w);
              a.bitmask[(static_cast<int64_t>(bo + i) * a.Hkv + g) * a.W + w] = word;
              if (word != 0u) atomicAdd(&cnt[iw], __popc(word));
            }
          }
          *slot = 0u;
        }
      }
    }
    epilogue_bar_sync();
    for (int x = m; x < nI; x += 128) a.counts[static_cast<int64_t>(bo + i0 + x) * a.Hkv + g] = cnt[x];
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
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
                                                      int64_t rows, const __grid_constant__ Fp2Plan P) {
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

size_t discover_smem_bytes(int D) { return D == 64 ? DiscCfg<64>::SMEM_BYTES : DiscCfg<128>::SMEM_BYTES; }

cudaError_t launch_discover(const DiscArgs& a, const Fp2Plan& P, int64_t items, int64_t rows, int32_t* row_ptr,
                            int32_t* col_idx, int64_t capacity, cudaStream_t stream) {
  cudaError_t e;
  if (a.D == 64) {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<64>), DiscCfg<64>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    discover_kernel<64><<<static_cast<unsigned>(items), DiscCfg<64>::THREADS, DiscCfg<64>::SMEM_BYTES, stream>>>(a, P);
  } else {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(discover_kernel<128>), DiscCfg<128>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    discover_kernel<128><<<static_cast<unsigned>(items), DiscCfg<128>::THREADS, DiscCfg<128>::SMEM_BYTES, stream>>>(a,
                                                                                                                 P);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scan_kernel<<<1, 1024, 0, stream>>>(a.counts, rows, row_ptr, capacity, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scatter_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(a.bitmask, a.W, row_ptr, col_idx, capacity,
                                                                           a.Hkv, rows, P);
  return cudaGetLastError();
}

}  // namespace fp2
