// Stage 2: exact sparse attention over the kept key blocks with mean correction for the
// pruned ones (FlashPrefill V2 paper page, Figure 3: the exact and mean-correction streams
// "merge inside the online softmax"; Figure 4: a pruned block J contributes
// |B_J| e^{s_J} (vbar_J, 1); Table 7: CSR per KV head, PackGQA).
//
// One CTA owns one (sequence r, query block i, KV head g, part) work item.  Its rows are
// the G query heads of group g packed against their shared KV head (PackGQA): an M tile is
// 128 rows = (128 / B) heads x B tokens, and a CTA carries NT <= 2 M tiles that share every
// K/V tile it loads.  The key stream of the row is
//     [virtual tiles][kept blocks in ascending order]
// where virtual tile v holds the pooled kbar/vbar of blocks [vB, vB + B): every pruned
// block j < i enters there as one extra "key" with logit q.kbar_j*scale + ln n_j, so the
// correction shares the exact path's MMAs and online softmax; kept blocks and blocks >= i
// are masked out of the virtual tiles.  The last kept block is the diagonal (causal mask).
//
// KV splits (count-balanced; paper page, Table 7).  Uniform: with few rows, each row's key stream
// is cut into `splits` contiguous ranges of equal tile count; every range is a separate CTA
// writing a normalised partial O and its LSE, merged afterwards by combine_kernel.  Adaptive:
// split_plan_kernel reads the index and cuts only the rows whose tile count exceeds the piece
// size into ranges ("pieces"); CTAs [0, adapt) of the launch run the pieces (long work first),
// the row CTAs of those rows exit at once, and the last piece of a (row, part) to finish merges
// the pieces' partials in its epilogue.
//
// Warp roles (384 threads = 3 warpgroups):
//   warps 0-3 / 4-7  softmax for M tile 0 / 1: one TMEM lane (row) per thread; read S (and
//                    release the S buffer at once), mask, online max with lazy O rescale
//                    (only when the running max grows past a threshold), write P (bf16, f32,
//                    or f16 for e4m3 inputs) to the tile's P columns in TMEM, and finally
//                    normalise O and write it (full blocks through a swizzled staging tile and
//                    TMA stores, partial blocks and KV-split partials with per-thread stores).
//   warp 8           producer: issues TMA loads of Q and the first key tiles, builds the
//                    kept-block bitmask, then loads the remaining K/V (or kbar/vbar) tiles into
//                    an NSLOT ring of shared-memory slots; finally prefetches into L2 the Q tiles
//                    of the CTA one wave ahead.
//   warp 9           QK issuer: S = Q_s K^T (SS form) into the shared S buffer.
//   warps 10, 11     PV issuers for M tiles 0 and 1: O_s += P_s V (A operand P_s read from TMEM).
//                    The products touch disjoint TMEM, so each is issued the moment its own
//                    inputs are ready and the tensor pipe interleaves them; one issuer would stall
//                    the pipe at every wait between groups.  An issuing warp delays the softmax
//                    warps of its SMSP (clock64 stamps: the quarter on the QK issuer's SMSP ends a
//                    tile ~800 cycles after the others), and one PV issuer per M tile on two more
//                    SMSPs measured fastest; giving each QK group its own warp as well was slower.
//                    All issue tcgen05.mma from lane 0 and signal mbarriers with tcgen05.commit.
//                    With one M tile warp 11 idles (it completes warpgroup 2 for the register
//                    split).
// e4m3 inputs: QK runs on the e4m3 Q and K tiles; V tiles come from the exact f16 copy of V that
// the pooling pass writes (and the mean-correction vbar tiles from its f16 means), so PV is an f16
// product with P written as f16.  Converting V here instead would redo it for every row that keeps
// a block (about 74 times per tile at 128K) on one warp's conversion pipe.
// TMEM: S | P0 | P1 | O0 | O1.  One S buffer serves both M tiles in turn: a softmax warpgroup
// copies its S tile into registers and releases the buffer before doing any arithmetic, so
// the next QK product (the other tile's, or this tile's next key tile) is computed while the
// softmax runs, and the tensor pipe never waits for a whole softmax between two products of
// the same tile.  P_s gets its own columns; the softmax writes P_s(j) only after PV_s(j-1)
// has read P_s(j-1).
#include <math_constants.h>

#include "fp2_device.cuh"
#include "fp2_kernels.h"

namespace fp2 {

#ifndef REG_LOW_T
#define REG_LOW_T 64
#endif

template <int DT, int D, int BN>
struct AttnCfg {
  static constexpr int ELT = DT == 0 ? 4 : (DT == 1 ? 2 : 1);
  static constexpr int KIND = DT == 0 ? 0 : (DT == 1 ? 1 : 2);
  static constexpr uint32_t FMT = DT == 0 ? 2u : (DT == 1 ? 1u : 0u);  // tf32 / bf16 / e4m3
  static constexpr int KCH = 128 / ELT;  // elements in one 128-byte swizzled row
  static constexpr int DCH = D / KCH;    // 128-byte chunks along d
  static constexpr int UK = 32 / ELT;    // K extent of one MMA instruction (32 bytes)
  static constexpr int BM = 128;
  static constexpr int Q_BYTES = BM * D * ELT;
  // e4m3: QK runs on e4m3 operands; the V side (V tiles and vbar tiles) is f16, PV an f16 MMA.
  static constexpr bool V16 = DT == 2;
  static constexpr int VELT = V16 ? 2 : ELT;        // bytes per V element
  static constexpr int VKCH = 128 / VELT;           // V elements in one 128-byte swizzled row
  static constexpr int VDCH = D / VKCH;             // 128-byte chunks of a V row
  static constexpr int K_BYTES = BN * D * ELT;      // one K (or kbar) tile
  static constexpr int V_BYTES = BN * D * VELT;     // one V (or vbar) tile
  static constexpr int KV_BYTES = K_BYTES > V_BYTES ? K_BYTES : V_BYTES;  // ring slot
  static constexpr int TILE_BUDGET = 200 * 1024;
  static constexpr int NSLOT_RAW = (TILE_BUDGET - 2 * Q_BYTES) / KV_BYTES;
  // Even, so that V loads (odd load indices) always land in odd slots: a V slot is released by
  // the PV products of both M tiles, issued from two warps.
  static constexpr int NSLOT = (NSLOT_RAW > 8 ? 8 : NSLOT_RAW) & ~1;
  // PV operand type: f16 for e4m3 inputs, else the input type; K extent of one PV MMA.
  static constexpr int PV_KIND = V16 ? 1 : KIND;
  static constexpr uint32_t PV_FMT = V16 ? 0u : FMT;  // kind::f16 format 0 = f16
  static constexpr int PV_UK = V16 ? 16 : UK;
  // P columns per M tile: one 32-bit column per key for f32, two keys per column for 16-bit P.
  static constexpr int PC = DT == 0 ? BN : BN / 2;
  static constexpr int S_COL = 0;
  static constexpr int P_COL0 = BN, P_COL1 = BN + PC;
  static constexpr int O_COL0 = BN + 2 * PC, O_COL1 = BN + 2 * PC + D;
  static constexpr int TMEM_COLS = 512;
  static constexpr int REG_LOW = REG_LOW_T;
  static constexpr int REG_HIGH = ((384 * 168 - 128 * REG_LOW) / 256) / 8 * 8 > 248
                                      ? 248 : ((384 * 168 - 128 * REG_LOW) / 256) / 8 * 8;
  static_assert(128 * REG_LOW + 256 * REG_HIGH <= 384 * 168, "register split exceeds the launch");
  // Online-softmax constants (log2 domain).  P is written as 2^(x - m + P_SHIFT); the running
  // max m is only raised when the row max grows by more than LAZY, so P <= 2^(P_SHIFT + LAZY).
  // e4m3 inputs (P in f16): P_SHIFT 4 keeps small probabilities further from f16's subnormal
  // range; 2^12 stays far below its 65504 maximum.
  static constexpr float P_SHIFT = DT == 2 ? 4.0f : 0.0f;
  static constexpr float LAZY = 8.0f;
  static constexpr uint32_t IDESC_S = make_idesc(FMT, FMT, 0, 0, 128, BN);
  static constexpr uint32_t IDESC_PV = make_idesc(PV_FMT, PV_FMT, 0, 1, 128, D);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NSLOT * KV_BYTES;
  static constexpr int NBAR = 2 + 2 * NSLOT + 2 + 2 + 2 + 2 + 2 + 2 + 2 + 2;
  // Output staging for TMA stores: tile s's normalised O (128 rows x d, output type) goes into
  // the shared memory of its own Q tile, free once the tile's last QK product is done; only when
  // it fits there (bf16 and f32 inputs; e4m3 Q tiles are half the size of a bf16 O tile).
  static constexpr int OUT_ELT = DT == 0 ? 4 : 2;
  static constexpr int OCH = 128 / OUT_ELT;          // output elements per 128-byte box row
  static constexpr int OBOX = BN * 128;              // one box: BN rows x 128 bytes
  static constexpr int O_STAGE_BYTES = 128 * D * OUT_ELT;
  static constexpr bool TMA_OUT = O_STAGE_BYTES <= Q_BYTES;
  static constexpr int OFF_MISC = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;
  static constexpr int OFF_MASK = OFF_MISC + 16;
  // Checked builds: hand-off counters (QK issues, S releases, P writes, PV issues per tile; loads
  // per ring slot), 16 words.
  static constexpr int OFF_CHK = OFF_MASK + FP2_MAX_BLOCKS / 8;
  // At least 116 KB so that a second CTA never shares the SM (each CTA holds all 512 TMEM columns).
  static constexpr int SMEM_RAW = OFF_CHK + 64 + 1024;
  static constexpr int SMEM_BYTES = SMEM_RAW > 116 * 1024 ? SMEM_RAW : 116 * 1024;
  static_assert(NSLOT >= 4, "K/V ring needs at least four slots (two key tiles in flight)");
  static_assert(O_COL1 + D <= TMEM_COLS, "TMEM budget");
  static_assert(OFF_BAR % 8 == 0 && OFF_MASK % 16 == 0 && OFF_CHK % 16 == 0 && NSLOT <= 8, "shared-memory layout");
  static_assert(D % KCH == 0 && BN % UK == 0 && D % 32 == 0 && BN % 32 == 0, "tile shape");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// tcgen05.ld of 32 columns followed by its wait, in one statement so that no use of the
// registers can be scheduled before the data has landed.
FP2_DEVICE void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// tcgen05.ld of 64 consecutive columns (2 x 32) followed by its wait, in one statement so
// that no use of the registers can be scheduled before the data has landed.
FP2_DEVICE void tmem_ld64_sync(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr + 0u), "r"(taddr + 32u)
      : "memory");
}

// tcgen05.ld of 128 consecutive columns (4 x 32) followed by its wait, in one statement so
// that no use of the registers can be scheduled before the data has landed.
FP2_DEVICE void tmem_ld128_sync(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%129];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95}, [%130];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%131];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr + 0u), "r"(taddr + 32u), "r"(taddr + 64u), "r"(taddr + 96u)
      : "memory");
}

// Bit e of the result is set when pooled block (base + e) is a pruned block of query block i:
// strictly left of the diagonal and absent from the kept set.
FP2_DEVICE uint32_t pruned_word(const uint32_t* kmask, int base, int i) {
  if (base >= i) return 0u;
  const uint32_t kept = kmask[base >> 5];
  const int nvalid = i - base;  // blocks base .. i-1 are candidates
  const uint32_t lim = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
  return ~kept & lim;
}

// Bounded wait used only while draining in-flight copies at exit; ignores the abort flag.
// Copies and MMAs complete within microseconds, so the limit is short (a fifth of the wait limit).
FP2_DEVICE void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      set_status(status, FP2_DEV_TIMEOUT);
      return;
    }
  }
}

template <int DT, int D, int BN>
__global__ void __launch_bounds__(384, 1)
    attention_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ Fp2Plan P) {
  using C = AttnCfg<DT, D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + C::NSLOT;
  uint64_t* s_full = kv_empty + C::NSLOT;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* mask_ready = o_done + 2;
  uint64_t* mma_done = mask_ready + 1;
  uint64_t* s_free = mma_done + 1;  // [2]: the S buffer has been copied out by softmax s
  uint64_t* pv_done = s_free + 2;   // [2]: PV issuer s's final commit
  uint64_t* o_staged = pv_done + 2; // [2]: every row of tile s is staged for the TMA store
  uint64_t* o_merge = o_staged + 2;    // [2]: piece CTAs: the tile's merge decision is in merge_flag
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);  // [2]
  uint32_t* kmask = reinterpret_cast<uint32_t*>(smem + C::OFF_MASK);
  // Checked builds: chk[s] QK_s issues, chk[2 + s] S releases by softmax s, chk[4 + s] P_s writes,
  // chk[6 + s] PV_s issues, chk[8 + k] loads into ring slot k.  Each is bumped by the signalling
  // thread before its arrive or commit; each waiter checks the exact count its own progress implies.
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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTAs [0, a.adapt) run the planned pieces of long rows (adaptive splits); the rest map to
  // (sequence, query block, KV head, part, split) in heavy-first order.
  int r, i, g, part, split, nsplit;
  const int item = static_cast<int>(blockIdx.x) < a.adapt ? static_cast<int>(blockIdx.x) : -1;
  if (item >= 0) {
    if (item >= *a.n_items) return;
    const int2 it = a.items[item];
    const int b = it.x / a.Hkv;
    g = it.x % a.Hkv;
    r = seq_of_block(P, b);
    i = b - P.blk_off[r];
    nsplit = it.y >> 16;
    part = (it.y >> 8) & 255;
    split = it.y & 255;
  } else {
    int sub;
    if (!map_heavy_first(P, 1, a.Hkv * a.parts * a.splits, blockIdx.x - a.adapt, r, i, sub)) return;
    nsplit = a.splits;
    split = sub % a.splits;
    g = (sub / a.splits) / a.parts;
    part = (sub / a.splits) % a.parts;
  }
  const int L = P.len[r];                 // query tokens of the sequence (or chunk)
  const int I = P.pre_blk[r] + i;         // absolute key block of query block i (the diagonal)
  const int Lk = P.pre_blk[r] * BN + L;   // key tokens of the sequence
  const int64_t row = static_cast<int64_t>(P.blk_off[r] + i) * a.Hkv + g;
  if (item < 0 && a.adapt > 0 && a.row_item0[row] >= 0) return;  // this row runs as pieces
  const int rs = a.row_ptr[row], re = a.row_ptr[row + 1];
  const int nkept = re - rs;
  if (nkept <= 0 || nkept > I + 1) {
    if (tid == 0) set_status(a.status, FP2_DEV_INDEX_OOB);
    return;
  }
  const int npruned = I + 1 - nkept;
  const int n_virt = (a.mean_correction && npruned > 0) ? (I + BN - 1) / BN : 0;
  const int n_tiles = n_virt + nkept;
  // Count-balanced KV split: this CTA takes key tiles [t_begin, t_end) of the row's stream.
  const int t_begin = static_cast<int>(static_cast<long long>(n_tiles) * split / nsplit);
  const int t_end = static_cast<int>(static_cast<long long>(n_tiles) * (split + 1) / nsplit);
  const int n_local = t_end - t_begin;

  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&o_done[s], 1);
      mbar_init(&s_free[s], 128);
      mbar_init(&o_staged[s], 128);
      mbar_init(&o_merge[s], 1);
    }
    for (int k = 0; k < C::NSLOT; ++k) {
      mbar_init(&kv_full[k], 1);
      // a V slot (odd) is released by both PV issuers when there are two M tiles
      mbar_init(&kv_empty[k], ((k & 1) && a.NT == 2) ? 2 : 1);
    }
    mbar_init(mask_ready, 1);
    mbar_init(mma_done, 1);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    *abort_flag = 0;
    if constexpr (FP2_CHECKED != 0)
      for (int k = 0; k < 16; ++k) chk[k] = 0u;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Register split: the launch gives 384 threads x 168 registers; warpgroup 2 (producer, MMA,
  // two idle warps) drops to REG_LOW and the two softmax warpgroups rise to REG_HIGH, with
  // 128 * REG_LOW + 256 * REG_HIGH <= 384 * 168 (checked at compile time).

  if (warp >= 8) {
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 8) {
      // ---------------------------------------------------------------- producer
      // Q and the first key tiles first (they need no mask), then the kept-block mask while
      // they are in flight, then the remaining key tiles as ring slots free up.
      // Load p of this CTA goes to slot p % NSLOT: K of tile t is load 2t, V load 2t+1.
      auto issue_kv = [&](int jt, int j, int q, int kv) {
        if (kv == 0 && (q >> 1) == a.withhold_k_tile) return;  // testing: this load never arrives
        const int slot = q % C::NSLOT;
        bump(8 + slot);
        if (q == a.miscount_load) bump(8 + slot);  // testing: a count the consumer does not expect
        // K side in the input type; V side in the PV operand type (f16 for e4m3 inputs).
        const int dch = kv ? C::VDCH : C::DCH, kch = kv ? C::VKCH : C::KCH;
        mbar_arrive_expect_tx(&kv_full[slot], kv ? C::V_BYTES : C::K_BYTES);
        uint8_t* dst = smem + C::OFF_KV + slot * C::KV_BYTES;
        if (j < 0) {
          const CUtensorMap* tm = kv ? &a.tm_vb : &a.tm_kb;
          for (int c = 0; c < dch; ++c)
            tma_load_3d(dst + c * (BN * 128), tm, &kv_full[slot], c * kch, g, P.k_blk_off[r] + jt * BN);
        } else if (a.page_table == nullptr || (kv && a.v_contig)) {
          const CUtensorMap* tm = kv ? &a.tm_v : &a.tm_k;
          for (int c = 0; c < dch; ++c)
            tma_load_3d(dst + c * (BN * 128), tm, &kv_full[slot], c * kch, g, P.k_tok_off[r] + j * BN);
        } else {
          const CUtensorMap* tm = kv ? &a.tm_v : &a.tm_k;
          const int PR = min(BN, a.page_size);
          for (int sb = 0; sb < BN / PR; ++sb) {
            int t = j * BN + sb * PR;
            if (t >= Lk) t = (Lk - 1) - ((Lk - 1) % PR);  // past the end: reload the last rows (masked)
            int page = a.page_table[static_cast<int64_t>(r) * a.max_pages + t / a.page_size];
            if (page < 0 || page >= a.num_pages) {
              set_status(a.status, FP2_DEV_PAGE_OOB);
              page = 0;
            }
            const int flat = page * a.page_size + (t % a.page_size);
            for (int c = 0; c < C::DCH; ++c)
              tma_load_3d(dst + c * (BN * 128) + sb * (PR * 128), tm, &kv_full[slot], c * C::KCH, g, flat);
          }
        }
      };
      // Tiles whose loads go out before the mask exists: as many as fit in the ring without a
      // release.  Their kept blocks come straight from the column list (clamped; the list is
      // validated below and a bad one is reported through the status word).
      const int npre = min(n_local, C::NSLOT / 2);
      if (lane == 0) {
        tma_prefetch_desc(&a.tm_q);
        tma_prefetch_desc(&a.tm_k);
        tma_prefetch_desc(&a.tm_v);
        tma_prefetch_desc(&a.tm_kb);
        tma_prefetch_desc(&a.tm_vb);
        constexpr int HS = 128 / BN;
        const int tokq = P.tok_off[r] + i * BN;
        for (int s = 0; s < a.NT; ++s) {
          mbar_arrive_expect_tx(&q_full[s], C::Q_BYTES);
          for (int hs = 0; hs < HS; ++hs) {
            const int hl = (part * a.NT + s) * HS + hs;
            const int h = g * a.G + (hl % a.G);
            for (int c = 0; c < C::DCH; ++c)
              tma_load_3d(smem + C::OFF_Q + s * C::Q_BYTES + c * (128 * 128) + hs * (BN * 128), &a.tm_q, &q_full[s],
                          c * C::KCH, h, tokq);
          }
        }
        for (int t = 0; t < npre; ++t) {
          const int jt = t_begin + t;
          const int j = jt < n_virt ? -1 : min(max(a.col_idx[rs + jt - n_virt], 0), I);
          issue_kv(jt, j, 2 * t, 0);
          issue_kv(jt, j, 2 * t + 1, 1);
        }
      }
      const int nw = (I + 32) / 32;
      for (int w = lane; w < nw; w += 32) kmask[w] = 0u;
      __syncwarp();
      bool bad = false;
      for (int e = lane; e < nkept; e += 32) {
        const int j = a.col_idx[rs + e];
        const int prev = e > 0 ? a.col_idx[rs + e - 1] : -1;
        if (j < 0 || j > I || j <= prev)
          bad = true;
        else if (fp2_check((j >> 5) < FP2_MAX_BLOCKS / 32, a.status))
          atomicOr(&kmask[j >> 5], 1u << (j & 31));
      }
      if (lane == 0 && a.col_idx[re - 1] != I) bad = true;
      if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(a.status, FP2_DEV_INDEX_OOB);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(mask_ready);
        // Kept blocks are taken in ascending order from the bit mask in shared memory (the same
        // sequence as the validated column list), so the loop below makes no global reads for
        // them.  It starts after the kept blocks of earlier splits and of the tiles issued above.
        const int nwords = (I >> 5) + 1;
        int wi = 0;
        uint32_t bits = kmask[0];
        int skip = max(t_begin + npre - n_virt, 0);
        while (wi + 1 < nwords && skip >= __popc(bits)) {
          skip -= __popc(bits);
          bits = kmask[++wi];
        }
        for (; skip > 0 && bits; --skip) bits &= bits - 1;
        auto next_kept = [&]() -> int {
          while (bits == 0 && wi + 1 < nwords) bits = kmask[++wi];
          if (bits == 0) return I;  // only after a rejected index (status already set)
          const int j = (wi << 5) + __ffs(bits) - 1;
          bits &= bits - 1;
          return j;
        };
        int p = 2 * npre;
        for (int jt = t_begin + npre; jt < t_end && !*abort_flag; ++jt) {
          const int j = jt >= n_virt ? next_kept() : -1;
          bool stop = false;
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = p % C::NSLOT, wrap = p / C::NSLOT;
            if (wrap > 0 && !mbar_wait(&kv_empty[slot], (wrap - 1) & 1, abort_flag, a.status, a.wait_limit_ns)) {
              stop = true;
              break;
            }
            issue_kv(jt, j, p, kv);
            ++p;
          }
          if (stop) break;
        }
        // The CTA that starts about one wave after this one (block index + grid SMs, in the
        // heavy-first order) will need its Q tiles first: bring them into L2 now.
        {
          int r2, i2, sub2;
          const long long v2 = static_cast<long long>(blockIdx.x) + a.num_sms - a.adapt;
          if (v2 >= 0 && map_heavy_first(P, 1, a.Hkv * a.parts * a.splits, v2, r2, i2, sub2)) {
            const int g2 = (sub2 / a.splits) / a.parts, part2 = (sub2 / a.splits) % a.parts;
            constexpr int HS2 = 128 / BN;
            for (int s = 0; s < a.NT; ++s)
              for (int hs = 0; hs < HS2; ++hs) {
                const int hl = (part2 * a.NT + s) * HS2 + hs;
                for (int c = 0; c < C::DCH; ++c)
                  tma_prefetch_l2_3d(&a.tm_q, c * C::KCH, g2 * a.G + (hl % a.G), P.tok_off[r2] + i2 * BN);
              }
          }
        }
        // Never leave with copies in flight.
        for (int s = 0; s < a.NT; ++s) mbar_wait_drain(&q_full[s], 0, a.status, a.wait_limit_ns / 5);
        for (int q = max(0, p - C::NSLOT); q < p; ++q) mbar_wait_drain(&kv_full[q % C::NSLOT], (q / C::NSLOT) & 1, a.status, a.wait_limit_ns / 5);
      }
    } else if (warp == 9 || warp == 10 || (warp == 11 && a.NT == 2)) {
      // ---------------------------------------------------------------- MMA issuers
      // QK issuer (warp 9), for key tile j with NT = 2: QK1(j) once softmax 0 has copied S0(j)
      // out, then QK0(j+1) once softmax 1 has copied S1(j) out; NT = 1: QK0(j+1) after S0(j).
      // PV issuers (warp 10 for M tile 0, warp 11 for M tile 1): PV_s(j) once P_s(j) is written.
      // Each warp runs its loop with warp-uniform control flow (every wait is voted) and lane 0
      // issues each tcgen05 instruction (the *_warp wrappers).
      {
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
          return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, a.status, a.wait_limit_ns));
        };
        // Loads come in the order K(0), V(0), K(1), V(1), ...: K(j) is load 2j, V(j) load 2j+1.
        auto slot_of = [&](int q) { return q % C::NSLOT; };
        auto kv_wait = [&](int q) {
          const bool got = wait_all(&kv_full[slot_of(q)], (q / C::NSLOT) & 1);
          if (got && lane == 0) expect(8 + slot_of(q), q / C::NSLOT + 1);  // the load of this use
          return got;
        };
        auto slot_addr = [&](int q) { return sbase + C::OFF_KV + slot_of(q) * C::KV_BYTES; };
        bool ok = true;
        if (warp == 9) {
          for (int s = 0; s < a.NT && ok; ++s) ok = wait_all(&q_full[s], 0);
          tc_fence_after();
          // Descriptors are formed once per tile; a K step only moves the start address, which is
          // the low 14 bits (address >> 4) of the descriptor and cannot carry (smem < 256 KB).
          auto issue_qk = [&](int s, uint32_t kaddr) {
            const uint64_t ad0 = smem_desc_sw128(sbase + C::OFF_Q + s * C::Q_BYTES, 16, 1024);
            const uint64_t bd0 = smem_desc_sw128(kaddr, 16, 1024);
            const uint32_t dcol = tmem + C::S_COL;
            // Fully unrolled with constant offsets and accumulate flags: a single warp then issues
            // back to back at the tensor rate (measured: one 128x128x16 MMA per 64 cycles), while
            // per-step descriptor arithmetic or a runtime flag costs 110-160 cycles per MMA.
#pragma unroll
            for (int k = 0; k < D / C::UK; ++k) {
              const int c = (k * C::UK) / C::KCH;
              const int koff = ((k * C::UK) % C::KCH) * C::ELT;
              umma_ss_warp<C::KIND>(dcol, ad0 + static_cast<uint64_t>((c * (128 * 128) + koff) >> 4),
                                    bd0 + static_cast<uint64_t>((c * (BN * 128) + koff) >> 4), C::IDESC_S,
                                    k > 0 ? 1u : 0u);
            }
            if (lane == 0) bump(s);
            __syncwarp();
            umma_commit_warp(&s_full[s]);
          };
          if (n_local > 0 && ok) {
            ok = kv_wait(0);
            if (ok) {
              tc_fence_after();
              issue_qk(0, slot_addr(0));
              if (a.NT == 1) umma_commit_warp(&kv_empty[slot_of(0)]);
            }
          }
          for (int jt = 0; jt < n_local && ok; ++jt) {  // jt: tile index within this split
            const int qk = 2 * jt;
            if (a.NT == 2) {
              if (!wait_all(&s_free[0], jt & 1)) break;  // softmax 0 holds S0(jt)
              if (lane == 0) expect(2, jt + 1);
              tc_fence_after();
              issue_qk(1, slot_addr(qk));
              umma_commit_warp(&kv_empty[slot_of(qk)]);  // K(jt) fully consumed
            }
            if (jt + 1 < n_local) {
              if (!kv_wait(qk + 2)) break;
              if (!wait_all(&s_free[a.NT - 1], jt & 1)) break;  // the last softmax holds its S(jt)
              if (lane == 0) expect(2 + a.NT - 1, jt + 1);
              tc_fence_after();
              issue_qk(0, slot_addr(qk + 2));
              if (a.NT == 1) umma_commit_warp(&kv_empty[slot_of(qk + 2)]);
            }
          }
          umma_commit_warp(mma_done);
          if (lane == 0) mbar_wait_drain(mma_done, 0, a.status, a.wait_limit_ns / 5);
          __syncwarp();
        } else {
          auto issue_pv = [&](int s, uint32_t vaddr, int jt) {
            const uint32_t pcol = tmem + (s ? C::P_COL1 : C::P_COL0);
            const uint32_t ocol = tmem + (s ? C::O_COL1 : C::O_COL0);
            // V is MN-major (d contiguous).  32-bit V uses the 32-byte-chunk swizzle with 4-row
            // atoms (SBO 512); 16-bit V the 16-byte-chunk swizzle with 8-row atoms.
            const uint64_t vd0 = DT == 0 ? smem_desc(vaddr, BN * 128, 512, 1u) : smem_desc_sw128(vaddr, BN * 128, 1024);
#pragma unroll
            for (int k = 0; k < BN / C::PV_UK; ++k) {
              const uint64_t bd = vd0 + static_cast<uint64_t>((k * C::PV_UK * 128) >> 4);
              umma_ts_warp<C::PV_KIND>(ocol, pcol + k * 8, bd, C::IDESC_PV, (jt > 0 || k > 0) ? 1u : 0u);
            }
            if (lane == 0) bump(6 + s);
            __syncwarp();
            umma_commit_warp(&o_done[s]);
          };
          // Warp 10 issues tile 0's products, warp 11 tile 1's: the two PV groups of a key tile
          // come from two warps on two SMSPs (an issuing warp slows the softmax warps of its SMSP).
          const int s = warp - 10;
          for (int jt = 0; jt < n_local && ok; ++jt) {
            const int qv = 2 * jt + 1;
            if (!(ok = kv_wait(qv))) break;
            if (!(ok = wait_all(&p_full[s], jt & 1))) break;
            if (lane == 0) expect(4 + s, jt + 1);
            tc_fence_after();
            issue_pv(s, slot_addr(qv), jt);
            umma_commit_warp(&kv_empty[slot_of(qv)]);  // this tile's share of V(jt) consumed
          }
          umma_commit_warp(&pv_done[s]);
          if (lane == 0) mbar_wait_drain(&pv_done[s], 0, a.status, a.wait_limit_ns / 5);
          __syncwarp();
        }
      }
    }
  } else {
    setmaxnreg_inc<C::REG_HIGH>();
    if (warp < 4 * a.NT) {
      // ---------------------------------------------------------------- softmax / epilogue
      const int s = warp >> 2, qd = warp & 3;
      const int rt = qd * 32 + lane;
      constexpr int HS = 128 / BN;
      const int hs = rt / BN, tl = rt % BN;
      const int hl = (part * a.NT + s) * HS + hs;
      const bool in_seq = (hl < a.G) && (i * BN + tl < L);
      const int h = g * a.G + min(hl, a.G - 1);
      // a row of the sequence whose output position lies inside O (the bound is checked in
      // checked builds)
      const bool row_ok = in_seq && fp2_check(P.tok_off[r] + i * BN + tl < a.total_tokens && h < a.Hq, a.status);
      const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
      const uint32_t s_addr = tmem + lane_base + C::S_COL;
      const uint32_t p_addr = tmem + lane_base + (s ? C::P_COL1 : C::P_COL0);
      const uint32_t o_addr = tmem + lane_base + (s ? C::O_COL1 : C::O_COL0);
      const float s2 = a.sm_scale_log2;
      const float bias_raw = a.log2_blk / s2;
      float m_run = -CUDART_INF_F, l_run = 0.f;
      bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(mask_ready, 0, abort_flag, a.status, a.wait_limit_ns));

      int done_tiles = 0;
      for (int jl = 0; jl < n_local && ok; ++jl) {
        const int jt = t_begin + jl;  // position in the row's key stream
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[s], jl & 1, abort_flag, a.status, a.wait_limit_ns));
        if (!ok) break;
        if (rt == 0) expect(s, jl + 1);  // QK_s(jl) and nothing later
        tc_fence_after();
        // The whole S row of this thread, in registers.
        uint32_t v[BN];
        if constexpr (BN == 128)
          tmem_ld128_sync(s_addr, v);
        else
          tmem_ld64_sync(s_addr, v);
        // S is in registers: hand the buffer to the next QK product.
        if (rt == 0) bump(2 + s);
        tc_fence_before();
        mbar_arrive(&s_free[s]);
        // PV_s(jl-1) must be complete before O_s is rescaled or P_s is overwritten.
        bool pv_prev_done = jl == 0;
        auto wait_pv_prev = [&]() {
          if (!pv_prev_done) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&o_done[s], (jl - 1) & 1, abort_flag, a.status, a.wait_limit_ns));
            if (ok && rt == 0) expect(6 + s, jl);  // PV_s(jl-1) and nothing later
            tc_fence_after();
            pv_prev_done = true;
          }
          return ok;
        };
        // Tile kinds: virtual (pooled keys of blocks [jt*BN, jt*BN+BN): only pruned blocks, with the
        // ln n_j bias), diagonal (causal mask), full (no mask).  The mask works on raw S values:
        // x = S * s2 with s2 > 0, so the bias is added as log2(n)/s2 and the max is taken on raw S.
        float xs[BN];
        if (jt < n_virt) {
          // The column mask and bias of a virtual tile are the same for every row of the CTA:
          // lane l of each warp works out the bias of columns l, l + 32, ... (+log2(n)/s2 for a
          // pruned block, -inf otherwise) and every row gets them by warp shuffles.
  #pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            const int blk = jt * BN + c * 32 + lane;
            const bool pr = blk < I && !((kmask[blk >> 5] >> (blk & 31)) & 1u);
            const float bias_l = pr ? bias_raw : -CUDART_INF_F;
  #pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 x2 = __fadd2_rn(
                  make_float2(__uint_as_float(v[c * 32 + e]), __uint_as_float(v[c * 32 + e + 1])),
                  make_float2(__shfl_sync(0xFFFFFFFFu, bias_l, e), __shfl_sync(0xFFFFFFFFu, bias_l, e + 1)));
              xs[c * 32 + e] = x2.x;
              xs[c * 32 + e + 1] = x2.y;
            }
          }
        } else if (jt == n_tiles - 1) {
  #pragma unroll
          for (int e = 0; e < BN; ++e) xs[e] = (e <= tl) ? __uint_as_float(v[e]) : -CUDART_INF_F;
        } else {
  #pragma unroll
          for (int e = 0; e < BN; ++e) xs[e] = __uint_as_float(v[e]);
        }
        // Row max with three-operand max, four independent chains.
        float m4[4];
  #pragma unroll
        for (int u = 0; u < 4; ++u) m4[u] = fmaxf(xs[2 * u], xs[2 * u + 1]);
  #pragma unroll
        for (int e = 8; e < BN; e += 8) {
  #pragma unroll
          for (int u = 0; u < 4; ++u) m4[u] = fmax3(m4[u], xs[e + 2 * u], xs[e + 2 * u + 1]);
        }
        const float mt = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * s2;
        const float m_new = fmaxf(m_run, mt);
        const bool need = m_new > m_run + C::LAZY;
        if (jl > 0 && __any_sync(0xFFFFFFFFu, need)) {
          if (!wait_pv_prev()) break;
          const float f = need ? fast_exp2(m_run - m_new) : 1.0f;
  #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32_sync(o_addr + c * 32, o);
  #pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 r2 = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                                           make_float2(f, f));
              o[e] = __float_as_uint(r2.x);
              o[e + 1] = __float_as_uint(r2.y);
            }
            tmem_st32(o_addr + c * 32, o);
          }
          tmem_st_wait();
        }
        if (need) {
          l_run = (m_run == -CUDART_INF_F) ? 0.f : l_run * fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(S*s2 - m + P_SHIFT), packed to the MMA operand type and written to P_s in TMEM.
        const float nmu = C::P_SHIFT - ((m_run == -CUDART_INF_F) ? 0.f : m_run);
        // Exponent arguments x * s2 + nmu and the row sums in packed f32x2 arithmetic (pairs of
        // adjacent scores); the same fused multiply-add as the scalar form, so P is unchanged.
        const float2 s22 = make_float2(s2, s2), nmu2 = make_float2(nmu, nmu);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        auto exp_pair = [&](int e2) -> float2 {
          const float2 t = __ffma2_rn(make_float2(xs[2 * e2], xs[2 * e2 + 1]), s22, nmu2);
          const float2 p = make_float2(fast_exp2(t.x), fast_exp2(t.y));
          acc[e2 & 1] = __fadd2_rn(acc[e2 & 1], p);
          return p;
        };
        if constexpr (DT == 1) {
          // 64 scores -> 32 packed words -> one TMEM store, chunk by chunk (keeps fewer P words live).
  #pragma unroll
          for (int c = 0; c < BN / 64; ++c) {
            uint32_t pk[32];
  #pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float2 p = exp_pair(c * 32 + e);
              pk[e] = pack_bf16x2(p.x, p.y);
            }
            if (c == 0 && !wait_pv_prev()) break;
            tmem_st32(p_addr + c * 32, pk);
          }
        } else if constexpr (DT == 2) {
          // f16 P for the f16 PV product: 64 scores -> 32 packed words -> one TMEM store.
  #pragma unroll
          for (int c = 0; c < BN / 64; ++c) {
            uint32_t pk[32];
  #pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float2 p = exp_pair(c * 32 + e);
              pk[e] = pack_f16x2(p.x, p.y);
            }
            if (c == 0 && !wait_pv_prev()) break;
            tmem_st32(p_addr + c * 32, pk);
          }
        } else {
          uint32_t pk[BN];
  #pragma unroll
          for (int e = 0; e < BN / 2; ++e) {
            const float2 p = exp_pair(e);
            pk[2 * e] = __float_as_uint(p.x);
            pk[2 * e + 1] = __float_as_uint(p.y);
          }
          if (wait_pv_prev()) {
  #pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_st32(p_addr + c * 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[c * 32]));
          }
        }
        if (!ok) break;
        const float rsum = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
        tmem_st_wait();
        if (rt == 0) bump(4 + s);
        tc_fence_before();
        mbar_arrive(&p_full[s]);
        l_run += rsum;
        done_tiles = jl + 1;
      }
      if (ok && done_tiles == n_local && n_local > 0)
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&o_done[s], (n_local - 1) & 1, abort_flag, a.status, a.wait_limit_ns));
      if (ok && n_local > 0 && rt == 0) expect(6 + s, n_local);
      tc_fence_after();
      if (item >= 0) {
        // Piece of a split row: its normalised partial O (fp32) and natural-log LSE go to the
        // piece's slot; the last piece of the (row, part) to finish, found with an atomic counter
        // per M tile, merges all of them with weights exp(LSE - max LSE) and writes the output
        // rows.  No CTA waits for another.  A piece with no visible key contributes LSE = -inf.
        const int prow = a.NT * 128;
        const int64_t srow = static_cast<int64_t>(item) * prow + s * 128 + rt;
        const bool slot_ok = fp2_check(srow < static_cast<int64_t>(a.adapt) * prow, a.status);  // checked builds
        const bool any = ok && n_local > 0 && l_run > 0.f;
        const float inv = any ? a.v_descale / l_run : 0.f;
        float* op = a.o_slot + srow * D;
  #pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (ok && n_local > 0) {
            tmem_ld32_sync(o_addr + c * 32, v);
          } else {
  #pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          float4* dst = reinterpret_cast<float4*>(op + c * 32);
          if (slot_ok) {
  #pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                   __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
          }
        }
        if (slot_ok)
          a.lse_slot[srow] = any ? (m_run + log2f(l_run) - C::P_SHIFT) * 0.6931471805599453f : -CUDART_INF_F;
        __threadfence();
        mbar_arrive(&o_staged[s]);
        const int first = item - split;  // first piece of this (row, part)
        if (qd == 0 && lane == 0) {
          int last = 0;
          if (mbar_wait(&o_staged[s], 0, abort_flag, a.status, a.wait_limit_ns)) {
            __threadfence();
            last = atomicAdd(&a.piece_cnt[first * 2 + s], 1) == nsplit - 1;
          }
          merge_flag[s] = last;
          mbar_arrive(&o_merge[s]);
        }
        const bool merge =
            __all_sync(0xFFFFFFFFu, mbar_wait(&o_merge[s], 0, abort_flag, a.status, a.wait_limit_ns)) && merge_flag[s] != 0;
        if (merge && row_ok) {
          __threadfence();
          const float* lp = a.lse_slot + static_cast<int64_t>(first) * prow + s * 128 + rt;
          const float* obase = a.o_slot + (static_cast<int64_t>(first) * prow + s * 128 + rt) * D;
          float m = -CUDART_INF_F;
          for (int k = 0; k < nsplit; ++k) m = fmaxf(m, __ldcg(lp + static_cast<int64_t>(k) * prow));
          float wsum = 0.f;
          for (int k = 0; k < nsplit; ++k) {
            const float l = __ldcg(lp + static_cast<int64_t>(k) * prow);
            wsum += l == -CUDART_INF_F ? 0.f : expf(l - m);
          }
          const float winv = wsum > 0.f ? 1.f / wsum : 0.f;
          const int tok = P.tok_off[r] + i * BN + tl;
  #pragma unroll 1
          for (int c = 0; c < D / 8; ++c) {  // eight output columns at a time
            float acc8[8];
  #pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] = 0.f;
            for (int k = 0; k < nsplit; ++k) {
              const float l = __ldcg(lp + static_cast<int64_t>(k) * prow);
              const float w = l == -CUDART_INF_F ? 0.f : expf(l - m);
              const float4* src = reinterpret_cast<const float4*>(obase + static_cast<int64_t>(k) * prow * D + c * 8);
              const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
              acc8[0] = fmaf(w, x0.x, acc8[0]);
              acc8[1] = fmaf(w, x0.y, acc8[1]);
              acc8[2] = fmaf(w, x0.z, acc8[2]);
              acc8[3] = fmaf(w, x0.w, acc8[3]);
              acc8[4] = fmaf(w, x1.x, acc8[4]);
              acc8[5] = fmaf(w, x1.y, acc8[5]);
              acc8[6] = fmaf(w, x1.z, acc8[6]);
              acc8[7] = fmaf(w, x1.w, acc8[7]);
            }
            const int64_t o_off = (static_cast<int64_t>(tok) * a.Hq + h) * D + c * 8;
            if constexpr (DT == 0) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + o_off);
              dst[0] = make_float4(acc8[0] * winv, acc8[1] * winv, acc8[2] * winv, acc8[3] * winv);
              dst[1] = make_float4(acc8[4] * winv, acc8[5] * winv, acc8[6] * winv, acc8[7] * winv);
            } else {
              uint4 w;
              w.x = pack_bf16x2(acc8[0] * winv, acc8[1] * winv);
              w.y = pack_bf16x2(acc8[2] * winv, acc8[3] * winv);
              w.z = pack_bf16x2(acc8[4] * winv, acc8[5] * winv);
              w.w = pack_bf16x2(acc8[6] * winv, acc8[7] * winv);
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + o_off) = w;
            }
          }
          if (a.lse != nullptr) a.lse[static_cast<int64_t>(h) * a.total_tokens + tok] = m + logf(wsum);
        }
      } else if (ok && a.splits > 1) {
        // Partial result of this split: normalised O (fp32) and its natural-log LSE, merged by
        // combine_kernel.  A split with no key tile (or no visible key for this row) contributes
        // O = 0 with LSE = -inf.
        const int tok = P.tok_off[r] + i * BN + tl;
        const bool any = n_local > 0 && l_run > 0.f;
        const float inv = any ? a.v_descale / l_run : 0.f;
        float* op = a.o_part + ((static_cast<int64_t>(split) * a.total_tokens + tok) * a.Hq + h) * D;
  #pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (n_local > 0) {
            tmem_ld32_sync(o_addr + c * 32, v);
          } else {
  #pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(op + c * 32);
  #pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                   __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
          }
        }
        if (row_ok)
          a.lse_part[(static_cast<int64_t>(split) * a.Hq + h) * a.total_tokens + tok] =
              any ? (m_run + log2f(l_run) - C::P_SHIFT) * 0.6931471805599453f : -CUDART_INF_F;
      } else if (C::TMA_OUT && a.o_tma && i * BN + BN <= L) {
        // Full block: every thread writes its normalised row into the tile's staging buffer in
        // the 128-byte-swizzled box layout of tm_o (16-byte chunk c of box row t at c ^ (t & 7)),
        // then one thread stores the boxes with TMA once all 128 rows are staged.  All threads
        // arrive on o_staged whatever happened before, so the bounded wait below always ends.
        uint8_t* stg = smem + C::OFF_Q + s * C::Q_BYTES;  // inside tile s's own Q buffer
        if (ok) {
          const float inv = a.v_descale / l_run;
  #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32_sync(o_addr + c * 32, v);
  #pragma unroll
            for (int q = 0; q < 32 * C::OUT_ELT / 16; ++q) {
              uint4 w;
              if constexpr (DT == 0) {
                w = make_uint4(__float_as_uint(__uint_as_float(v[4 * q]) * inv),
                               __float_as_uint(__uint_as_float(v[4 * q + 1]) * inv),
                               __float_as_uint(__uint_as_float(v[4 * q + 2]) * inv),
                               __float_as_uint(__uint_as_float(v[4 * q + 3]) * inv));
              } else {
                w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
              }
              const int off = c * 32 * C::OUT_ELT + q * 16;  // byte offset of this chunk in the row
              const int k = off / 128, ci = (off % 128) / 16;
              *reinterpret_cast<uint4*>(stg + (k * HS + hs) * C::OBOX + tl * 128 + ((ci ^ (tl & 7)) * 16)) = w;
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&o_staged[s]);
        if (qd == 0 && lane == 0 && mbar_wait(&o_staged[s], 0, abort_flag, a.status, a.wait_limit_ns) && !*abort_flag) {
          const int tok0 = P.tok_off[r] + i * BN;
          for (int hs2 = 0; hs2 < HS; ++hs2) {
            const int hl2 = (part * a.NT + s) * HS + hs2;
            if (hl2 >= a.G) continue;
            for (int k = 0; k < D / C::OCH; ++k)
              tma_store_3d(&a.tm_o, stg + (k * HS + hs2) * C::OBOX, k * C::OCH, g * a.G + hl2, tok0);
          }
          bulk_commit_group();
          bulk_wait_read_all();
        }
        if (ok && row_ok && a.lse != nullptr)
          a.lse[static_cast<int64_t>(h) * a.total_tokens + P.tok_off[r] + i * BN + tl] =
              (m_run + log2f(l_run) - C::P_SHIFT) * 0.6931471805599453f;
      } else if (ok) {
        const int tok = P.tok_off[r] + i * BN + tl;
        const float inv = a.v_descale / l_run;
  #pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_sync(o_addr + c * 32, v);
          if (row_ok) {
            if constexpr (DT == 0) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) +
                                                      (static_cast<int64_t>(tok) * a.Hq + h) * D + c * 32);
  #pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                     __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                    (static_cast<int64_t>(tok) * a.Hq + h) * D + c * 32);
  #pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * inv, __uint_as_float(v[8 * e + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * inv, __uint_as_float(v[8 * e + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * inv, __uint_as_float(v[8 * e + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * inv, __uint_as_float(v[8 * e + 7]) * inv);
                dst[e] = w;
              }
            }
          }
        }
        if (row_ok && a.lse != nullptr)
          a.lse[static_cast<int64_t>(h) * a.total_tokens + tok] =
              (m_run + log2f(l_run) - C::P_SHIFT) * 0.6931471805599453f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Adaptive count-balanced splits (paper page, Table 7: "count-balanced CSR splits"), planned on
// the device from the index, so the host needs no copy of it.  One CTA sizes every row in key
// tiles as the attention kernel streams them (virtual tiles of the mean correction + kept
// blocks), picks the piece size T (piece_tiles, or the launch's total tile work over 4 x SMs, at
// least 32), and lists min(64, ceil(tiles / T)) pieces for every part of each row longer than T,
// rows in index order, while they fit in a.adapt.  The pieces of one (row, part) are consecutive.
constexpr int kPlanSmemRows = 32768;  // rows whose tile counts the plan keeps in shared memory

__global__ void __launch_bounds__(1024) split_plan_kernel(const __grid_constant__ AttnArgs a,
                                                          const __grid_constant__ Fp2Plan P, int64_t rows, int BN,
                                                          int piece_tiles) {
  extern __shared__ int32_t tiles_s[];  // [rows] when rows <= kPlanSmemRows
  __shared__ long long red[32];
  __shared__ int n_used;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool cached = rows <= kPlanSmemRows;
  auto row_tiles = [&](int64_t x) {
    const int b = static_cast<int>(x / a.Hkv);
    int lo = 0, hi = P.num_seqs - 1;  // the last sequence whose first block is <= b
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P.blk_off[mid] <= b) lo = mid; else hi = mid - 1;
    }
    const int I = P.pre_blk[lo] + (b - P.blk_off[lo]);
    const int nk = max(0, min(a.row_ptr[x + 1] - a.row_ptr[x], I + 1));
    const int nv = (a.mean_correction && I + 1 - nk > 0) ? (I + BN - 1) / BN : 0;
    return nv + nk;
  };
  for (int k = tid; k < a.adapt * 2; k += 1024) a.piece_cnt[k] = 0;
  if (tid == 0) n_used = 0;
  // Pass 1, coalesced: every row's tile count (kept in shared memory) and their sum.
  long long loc = 0;
  for (int64_t x = tid; x < rows; x += 1024) {
    const int t = row_tiles(x);
    if (cached) tiles_s[x] = t;
    loc += t;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) loc += __shfl_xor_sync(0xFFFFFFFFu, loc, o);
  if (lane == 0) red[warp] = loc;
  __syncthreads();
  long long total = 0;
  for (int w = 0; w < 32; ++w) total += red[w];
  __syncthreads();
  long long T = piece_tiles;
  if (T <= 0) {
    const long long slots = 4LL * max(a.num_sms, 1);
    T = max(32LL, (total * a.parts + slots - 1) / slots);
  }
  auto pieces_of = [&](int t) { return t > T ? static_cast<int>(min(64LL, (t + T - 1) / T)) : 1; };
  // Pass 2: exclusive scan of the piece counts (pieces x parts of each split row) over contiguous
  // row segments, then the piece list.
  const int64_t seg = (rows + 1023) / 1024;
  const int64_t s0 = min(rows, tid * seg), s1 = min(rows, s0 + seg);
  long long cnt_loc = 0;
  for (int64_t x = s0; x < s1; ++x) {
    const int S = pieces_of(cached ? tiles_s[x] : row_tiles(x));
    if (S > 1) cnt_loc += static_cast<long long>(S) * a.parts;
  }
  long long incl = cnt_loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  long long base = incl - cnt_loc;
  for (int w = 0; w < warp; ++w) base += red[w];
  int used = 0;
  for (int64_t x = s0; x < s1; ++x) {
    const int S = pieces_of(cached ? tiles_s[x] : row_tiles(x));
    const long long cnt = S > 1 ? static_cast<long long>(S) * a.parts : 0;
    if (cnt > 0 && base + cnt <= a.adapt) {
      a.row_item0[x] = static_cast<int32_t>(base);
      for (int pt = 0; pt < a.parts; ++pt)
        for (int k = 0; k < S; ++k)
          a.items[base + pt * S + k] = make_int2(static_cast<int>(x), (S << 16) | (pt << 8) | k);
      used = static_cast<int>(base + cnt);
    } else {
      a.row_item0[x] = -1;
    }
    base += cnt;
  }
  atomicMax(&n_used, used);
  __syncthreads();
  if (tid == 0) *a.n_items = n_used;
}

cudaError_t launch_split_plan(const AttnArgs& a, const Fp2Plan& P, int64_t rows, int B, int piece_tiles,
                              cudaStream_t stream) {
  const int smem = static_cast<int>(std::min<int64_t>(rows, kPlanSmemRows) * 4);
  const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(split_plan_kernel), smem);
  if (e != cudaSuccess) return e;
  split_plan_kernel<<<1, 1024, smem, stream>>>(a, P, rows, B, piece_tiles);
  return cudaGetLastError();
}

// Merge of the KV-split partials: for every (token, head), O = sum_s w_s O_s / sum_s w_s and
// LSE = m + ln sum_s w_s with w_s = exp(LSE_s - m), m = max_s LSE_s.  One warp per row, each lane
// owning D/32 consecutive-by-lane columns (coalesced).
template <int D, bool F32OUT>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ lse_part, int S, int T, int Hq,
                                                      void* out, float* lse) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= static_cast<int64_t>(T) * Hq) return;
  const int t = static_cast<int>(row / Hq), h = static_cast<int>(row % Hq);
  float m = -CUDART_INF_F;
  for (int s = 0; s < S; ++s) m = fmaxf(m, lse_part[(static_cast<int64_t>(s) * Hq + h) * T + t]);
  float acc[D / 32];
#pragma unroll
  for (int k = 0; k < D / 32; ++k) acc[k] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < S; ++s) {
    const float l = lse_part[(static_cast<int64_t>(s) * Hq + h) * T + t];
    const float w = (l == -CUDART_INF_F) ? 0.f : expf(l - m);
    wsum += w;
    const float* src = o_part + ((static_cast<int64_t>(s) * T + t) * Hq + h) * D;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) acc[k] = fmaf(w, src[lane + 32 * k], acc[k]);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {
    const int64_t idx = (static_cast<int64_t>(t) * Hq + h) * D + lane + 32 * k;
    if constexpr (F32OUT)
      static_cast<float*>(out)[idx] = acc[k] * inv;
    else
      static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(acc[k] * inv);
  }
  if (lse != nullptr && lane == 0) lse[static_cast<int64_t>(h) * T + t] = m + logf(wsum);
}

cudaError_t launch_combine(int dtype, int D, const float* o_part, const float* lse_part, int S, int T, int Hq,
                           void* out, float* lse, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(T) * Hq;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  const bool f32 = dtype == FP2_F32;
  if (D == 64 && f32)
    combine_kernel<64, true><<<blocks, 256, 0, stream>>>(o_part, lse_part, S, T, Hq, out, lse);
  else if (D == 64)
    combine_kernel<64, false><<<blocks, 256, 0, stream>>>(o_part, lse_part, S, T, Hq, out, lse);
  else if (f32)
    combine_kernel<128, true><<<blocks, 256, 0, stream>>>(o_part, lse_part, S, T, Hq, out, lse);
  else
    combine_kernel<128, false><<<blocks, 256, 0, stream>>>(o_part, lse_part, S, T, Hq, out, lse);
  return cudaGetLastError();
}

template <int DT, int D, int BN>
static cudaError_t launch_one(const AttnArgs& a, const Fp2Plan& P, int64_t items, cudaStream_t stream) {
  using C = AttnCfg<DT, D, BN>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(attention_kernel<DT, D, BN>), C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  attention_kernel<DT, D, BN><<<static_cast<unsigned>(items), 384, C::SMEM_BYTES, stream>>>(a, P);
  return cudaGetLastError();
}

size_t attention_smem_bytes(int dtype, int D, int B) {
  if (dtype == FP2_F32 && D == 64 && B == 64) return AttnCfg<0, 64, 64>::SMEM_BYTES;
  if (dtype == FP2_F32 && D == 64 && B == 128) return AttnCfg<0, 64, 128>::SMEM_BYTES;
  if (dtype == FP2_BF16 && D == 64 && B == 64) return AttnCfg<1, 64, 64>::SMEM_BYTES;
  if (dtype == FP2_BF16 && D == 64 && B == 128) return AttnCfg<1, 64, 128>::SMEM_BYTES;
  if (dtype == FP2_BF16 && D == 128 && B == 64) return AttnCfg<1, 128, 64>::SMEM_BYTES;
  if (dtype == FP2_BF16 && D == 128 && B == 128) return AttnCfg<1, 128, 128>::SMEM_BYTES;
  if (dtype == FP2_E4M3 && D == 128 && B == 64) return AttnCfg<2, 128, 64>::SMEM_BYTES;
  if (dtype == FP2_E4M3 && D == 128 && B == 128) return AttnCfg<2, 128, 128>::SMEM_BYTES;
  return 0;
}

cudaError_t launch_attention(int dtype, int D, int B, const AttnArgs& a, const Fp2Plan& P, int64_t items,
                             cudaStream_t stream) {
  if (dtype == FP2_F32 && D == 64 && B == 64) return launch_one<0, 64, 64>(a, P, items, stream);
  if (dtype == FP2_F32 && D == 64 && B == 128) return launch_one<0, 64, 128>(a, P, items, stream);
  if (dtype == FP2_BF16 && D == 64 && B == 64) return launch_one<1, 64, 64>(a, P, items, stream);
  if (dtype == FP2_BF16 && D == 64 && B == 128) return launch_one<1, 64, 128>(a, P, items, stream);
  if (dtype == FP2_BF16 && D == 128 && B == 64) return launch_one<1, 128, 64>(a, P, items, stream);
  if (dtype == FP2_BF16 && D == 128 && B == 128) return launch_one<1, 128, 128>(a, P, items, stream);
  if (dtype == FP2_E4M3 && D == 128 && B == 64) return launch_one<2, 128, 64>(a, P, items, stream);
  if (dtype == FP2_E4M3 && D == 128 && B == 128) return launch_one<2, 128, 128>(a, P, items, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fp2
