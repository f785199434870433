// Device helpers for sm_100a: mbarriers, TMA tile loads, tcgen05 (UMMA / TMEM)
// wrappers written directly in PTX, plus the heavy-first work-item mapping.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "fp2_plan.h"

#define FP2_DEVICE __device__ __forceinline__

namespace fp2 {

// ------------------------------------------------------------------ misc

FP2_DEVICE uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

FP2_DEVICE uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

FP2_DEVICE void set_status(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

// Checked builds (FP2_CHECKED=1): an invariant that does not hold sets FP2_DEV_CHECK and the caller
// skips the guarded access.  Normal builds compile every check away.
#ifndef FP2_CHECKED
#define FP2_CHECKED 0
#endif
FP2_DEVICE bool fp2_check(bool cond, uint32_t* status) {
  if constexpr (FP2_CHECKED != 0) {
    if (!cond) set_status(status, FP2_DEV_CHECK);
    return cond;
  } else {
    return true;
  }
}

// Work item v of a list ordered by level descending (level = query block or query-block tile),
// `width` items per (sequence, level), sequences with fewer levels dropping out as the level
// falls.  nlev(r) = ceil(nblk[r] / tile); tile is 1 or P.disc_tile (the two tables the host
// builds).  The segment of the k-th sequence in `sorted` order is found by binary search over
// its precomputed start.  Returns false when v is past the end.
FP2_DEVICE bool map_heavy_first(const Fp2Plan& P, int tile, int width, long long v, int& r, int& lvl, int& sub) {
  const int32_t* lb = tile == 1 ? P.lvl_base1 : P.lvl_base_t;
  const int n = P.num_seqs;
  if (v < 0 || v >= static_cast<long long>(lb[n]) * width) return false;
  int lo_k = 0, hi_k = n - 1;  // the last k with lb[k] * width <= v
  while (lo_k < hi_k) {
    const int mid = (lo_k + hi_k + 1) >> 1;
    if (static_cast<long long>(lb[mid]) * width <= v) lo_k = mid; else hi_k = mid - 1;
  }
  const int k = lo_k;
  const int hi = (P.nblk[P.sorted[k]] + tile - 1) / tile;
  const long long per_level = static_cast<long long>(k + 1) * width;
  const long long off = v - static_cast<long long>(lb[k]) * width;
  lvl = hi - 1 - static_cast<int>(off / per_level);
  const int rem = static_cast<int>(off % per_level);
  r = P.sorted[rem / width];
  sub = rem % width;
  return true;
}

// Sequence of query block b (the last sequence whose first block is <= b).
FP2_DEVICE int seq_of_block(const Fp2Plan& P, int b) {
  int lo = 0, hi = P.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.blk_off[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Sequence of key block b.
FP2_DEVICE int seq_of_key_block(const Fp2Plan& P, int b) {
  int lo = 0, hi = P.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.k_blk_off[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ mbarrier

FP2_DEVICE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
FP2_DEVICE void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
FP2_DEVICE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
FP2_DEVICE void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One probe of the phase; the thread may sleep in the probe for up to 0.5 ms and is woken as soon
// as the phase completes, so waiting threads do not burn issue slots.
FP2_DEVICE bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}

template <uint32_t N>
FP2_DEVICE void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
FP2_DEVICE void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Bounded wait: gives up after limit_ns of wall time (kWaitLimitNs unless the launch passes its
// own), or at once when another role of the CTA already gave up; records FP2_DEV_TIMEOUT and
// returns false.  Nothing in this library waits without a limit.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// Non-blocking probe of the phase (no suspend): the cheap first check of a wait that is often
// already satisfied.
FP2_DEVICE bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

FP2_DEVICE bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status,
                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_test_wait(bar, parity)) return true;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      set_status(status, FP2_DEV_TIMEOUT);
      return false;
    }
  }
}

// ------------------------------------------------------------------ TMA

FP2_DEVICE void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Bring a TMA box into L2 without a destination in shared memory.
FP2_DEVICE void tma_prefetch_l2_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

FP2_DEVICE void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// TMA tile store from shared memory (bulk-group completion).  Coordinates are never negative and
// the innermost one is a multiple of 16 bytes.
FP2_DEVICE void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
FP2_DEVICE void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store has finished reading its shared-memory source.
FP2_DEVICE void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the async (TMA) proxy.
FP2_DEVICE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05

FP2_DEVICE void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
FP2_DEVICE void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
FP2_DEVICE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
FP2_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FP2_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (sm100 encoding: version 1 at bit 46, layout type at bits
// 61-63: 2 = 128-byte swizzle of 16-byte chunks, 1 = 128-byte swizzle of 32-byte chunks, the
// only layout the tensor cores accept for MN-major 32-bit operands).  lbo/sbo in bytes.
FP2_DEVICE uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}
FP2_DEVICE uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) { return smem_desc(saddr, lbo, sbo, 2u); }

// Instruction descriptor: f32 accumulator, operand formats, majors, N and M.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t a_fmt, uint32_t b_fmt, uint32_t a_mn_major,
                                                  uint32_t b_mn_major, uint32_t M, uint32_t N) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// kind: 0 = tf32, 1 = f16 (bf16 operands), 2 = f8f6f4 (e4m3 operands)
template <int KIND>
FP2_DEVICE void umma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  } else if constexpr (KIND == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  }
}

// A operand read from tensor memory (row m in lane m, K packed along columns).
template <int KIND>
FP2_DEVICE void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  } else if constexpr (KIND == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
  }
}

// Arrive on an mbarrier once every tcgen05.mma issued so far by this thread has completed.
FP2_DEVICE void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Warp-collective forms: all 32 lanes of a converged warp call them with the same (warp-uniform)
// operands and lane 0 alone issues (predicate from %laneid inside the statement).  Keeping the
// issuing loop warp-uniform lets descriptors and addresses stay in uniform registers, so
// back-to-back MMAs issue without per-instruction register-to-uniform moves.  Lane 0 issues
// every MMA and every commit, so a commit tracks all of the warp's MMAs.
#define FP2_LANE0_PRED "{\n\t.reg .pred e, p;\n\t.reg .u32 l;\n\tmov.u32 l, %%laneid;\n\tsetp.eq.u32 e, l, 0;\n\t"
#define FP2_UMMA_WARP_SS(KINDSTR)                                                                  \
  asm volatile(FP2_LANE0_PRED "setp.ne.b32 p, %4, 0;\n\t"                                          \
               "@e tcgen05.mma.cta_group::1.kind::" KINDSTR " [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem), \
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)                                      \
               : "memory")
#define FP2_UMMA_WARP_TS(KINDSTR)                                                                  \
  asm volatile(FP2_LANE0_PRED "setp.ne.b32 p, %4, 0;\n\t"                                          \
               "@e tcgen05.mma.cta_group::1.kind::" KINDSTR " [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem), \
               "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)                                     \
               : "memory")

template <int KIND>
FP2_DEVICE void umma_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  if constexpr (KIND == 0)
    FP2_UMMA_WARP_SS("tf32");
  else if constexpr (KIND == 1)
    FP2_UMMA_WARP_SS("f16");
  else
    FP2_UMMA_WARP_SS("f8f6f4");
}
template <int KIND>
FP2_DEVICE void umma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  if constexpr (KIND == 0)
    FP2_UMMA_WARP_TS("tf32");
  else if constexpr (KIND == 1)
    FP2_UMMA_WARP_TS("f16");
  else
    FP2_UMMA_WARP_TS("f8f6f4");
}
FP2_DEVICE void umma_commit_warp(uint64_t* bar) {
  asm volatile(FP2_LANE0_PRED
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}
#undef FP2_UMMA_WARP_SS
#undef FP2_UMMA_WARP_TS
#undef FP2_LANE0_PRED

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets row (lane base + t).
FP2_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
FP2_DEVICE void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 16 consecutive columns (used for packed 16-bit / 8-bit P stores of short rows).
FP2_DEVICE void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// 8 consecutive columns (packed e4m3 P of 32 keys).
FP2_DEVICE void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
FP2_DEVICE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
FP2_DEVICE void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ numeric helpers

FP2_DEVICE float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (three-operand max.f32, sm_100).
FP2_DEVICE float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two floats -> packed bf16x2 (lo in the low half).
FP2_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Four floats -> packed e4m3x4 (v0 in the lowest byte), saturating.
FP2_DEVICE uint32_t pack_e4m3x4(float v0, float v1, float v2, float v3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(v1), "f"(v0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(v3), "f"(v2));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Two floats -> packed f16x2 (lo in the low half).
FP2_DEVICE uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// e4m3x2 (low byte = first value) -> f16x2 bits (first value in the low half), exact.
FP2_DEVICE uint32_t e4m3x2_to_f16x2(uint32_t v16) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(v16)));
  return h;
}



}  // namespace fp2
