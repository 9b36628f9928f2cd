// Spatial / full attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, per (b, t, head), O = softmax(Q K^T * scale) V over the S tokens
// of frame t (ScaleFusion review, "三、技术架构": the spatial layer; with T = 1
// it is the image-DiT full attention of the xDiT summary, section 3), or the
// normalised partial over one key range [kv0, kv1) plus its log-sum-exp, the
// per-chunk step of ring / Torus attention (SwiftFusion summary,
// Methodology 2).
//
// Design (one persistent CTA per SM, warp-specialised, 20 warps):
//   * A work item is 256 query rows of one (b, t, head) as two 128-row tiles
//     A and B; CTAs walk the items with a static stride.  Q tiles stay
//     resident in shared memory (double-buffered across items when they fit);
//     K and V tiles of 64 keys stream through a ring of TMA loads (warp 12).
//   * Tensor-core work runs on four issuer warps, one per (tile, product):
//     S = Q K^T into TMEM (fp32) for tile A (warp 13) and tile B (warp 14),
//     O += P V (warps 15 and 16) with P read straight from TMEM (the "TS"
//     form).  The four streams enter the tensor pipe independently, so no
//     stream waits behind another's MMAs that are held up by the shared-
//     memory reads they all share.  Registers are rebalanced per warpgroup
//     with setmaxnreg: the single-thread roles give theirs to the softmax.  S
//     is double-buffered per tile, so S of step j+1 is ready before the
//     softmax of step j ends; S(j+2) reuses the buffer of S(j) once PV(j) has
//     read P(j) from it.  The waits along this chain poll their barrier a few
//     times before sleeping (mbar_wait_spin).
//   * Ring mode (st_attn_ring): an item walks the R KV chunks from the one
//     holding its first row, carrying its running statistics across them;
//     the chunk edges come from host tables, and when every chunk is a whole
//     number of 64-key steps the walk is a plain rotation (RING = 2).
//   * Head dims 72/80 with long items keep Q in TMEM beside O (QTMEM), so S
//     becomes a TS product that reads only K from shared memory.
//   * Warps 0-3 (tile A) and 4-7 (tile B) are the softmax warpgroups: one
//     thread per query row (TMEM lane), 64 scores per step loaded with
//     tcgen05.ld, row max, exp2 with the softmax scale folded in (part of the
//     exponentials on the FMA pipe with a polynomial), row sum in fp32, P
//     packed to bf16 and written back over the S columns.  The running max is
//     only raised (and O rescaled in TMEM) when it grows by more than 2^8.
//   * Warps 8-11 are the epilogue warpgroup: once the last PV of a tile is
//     done they read O from TMEM, divide by the row sum handed over by the
//     softmax, round once to bf16 (or keep fp32 partials), stage 32 x 16
//     blocks in shared memory and write them with bulk tensor stores, plus the
//     natural-log LSE.  The softmax warps go straight on to the next item.
//   * Merge mode (st_attn_spatial_merge): the epilogue merges the chunk's
//     normalised O with the accumulated fp32 partial of earlier chunks,
//     o = w_a o_a + w_c O / l with w = exp(lse - M) / sum, and writes the
//     merged LSE.  For head dims up to 80 the copy engine stages the
//     accumulated rows of one tile in shared memory while the item runs;
//     larger head dims load them from global memory one chunk ahead.
//   * Head dims 32..128: Q and K split D into a 64-wide 128B-swizzled chunk and
//     a remainder chunk padded to 16/32/64 (zero-filled by TMA beyond D); V is
//     stored as column atoms so that PV is one instruction of N = padded D.
//   * Every wait on an mbarrier is bounded (wall clock).  A wait that runs out
//     records its site in a device error word, raises an abort epoch that
//     makes every other wait of the same launch give up, drains in-flight
//     copies and MMAs, frees TMEM and exits; the host reports ST_ERR_TIMEOUT.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "attn_geom.cuh"

namespace {

using st::pdl_trigger;
using st::pdl_wait;

__device__ unsigned int g_attn_error;        // sites of waits that ran out
__device__ unsigned int g_attn_abort_epoch;  // launch epoch that must abort

constexpr int NUM_THREADS = 640;             // 20 warps = 5 warpgroups
constexpr int BLOCK_M = 128;                 // query rows per tile
constexpr int BLOCK_N = 64;                  // keys per K/V tile (one softmax step)
constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s per wait
// warp roles (warps 0-7: softmax of tiles A and B)
constexpr int W_EPI = 8;                     // epilogue warpgroup: warps 8-11
constexpr int W_LOAD = 12;                   // TMA producer
constexpr int W_S0 = 13;                     // S issuer of tile A (tile B: W_S0 + 1); also allocates TMEM
constexpr int W_PV0 = 15;                    // PV issuer of tile A (tile B: W_PV0 + 1)
constexpr int W_ONES = 17;                   // writes the ones column into V tiles (padded head dims); 18-19 idle
// Registers per thread after the split (setmaxnreg): the launch gives every
// thread 96 (640 x 96 = 61440); the two softmax warpgroups and the epilogue
// take more, and the issuer / loader warpgroups give back:
// 256 x 128 + 128 x 128 + 256 x 48 = 61440 in general, and
// 256 x 152 + 128 x 96 + 256 x 40 = 61440 for head dims up to 80 without the
// merge, whose epilogue holds at most 80 columns of O (measured 2% faster at
// S = 1200 and 8160, D = 72; 1-2% slower at D = 128).
template <bool WIDE> struct RegSplit {
  static constexpr int SOFTMAX = WIDE ? 152 : 128, EPI = WIDE ? 96 : 128, ISSUE = WIDE ? 40 : 48;
  static_assert(256 * SOFTMAX + 128 * EPI + 256 * ISSUE <= NUM_THREADS * 96, "register split");
};
constexpr int EPI_COLS = 16;                 // O columns per staged store
constexpr int EPI_BUF = 32 * EPI_COLS * 4;   // bytes of one staging buffer (32 rows, fp32)
// TMEM columns: per tile two S buffers of BLOCK_N fp32 columns, then O.
constexpr int TM_O = 256;                    // O(tile X) at TM_O + X * 128

template <int D, bool MERGE = false, bool QTMEM = false> struct Cfg {
  static constexpr int C0 = D >= 64 ? 64 : 32;
  static constexpr int R1 = D > 64 ? D - 64 : 0;
  static constexpr int C1 = R1 == 0 ? 0 : (R1 <= 16 ? 16 : (R1 <= 32 ? 32 : 64));
  static constexpr int DP = C0 + C1;                   // padded head dim of Q and K
  static constexpr int SW0 = C0 * 2, SW1 = C1 * 2;     // row bytes = swizzle span
  static constexpr int QT0 = BLOCK_M * SW0, QT1 = BLOCK_M * SW1;
  static constexpr int QTILE = QT0 + QT1;              // bytes of one Q tile (128 rows)
  static constexpr int KT0 = BLOCK_N * SW0, KT1 = BLOCK_N * SW1;
  static constexpr int KTILE = KT0 + KT1;              // bytes of one K tile (64 keys)
  // V is stored as DPV / VW column atoms of VW elements (MN-major for PV), so
  // that O += P V is one instruction with N = DPV per 16 keys.
  static constexpr int VW = (D == 72 || D == 80) ? 16 : ((D == 96 || D == 32) ? 32 : 64);
  static constexpr int DPV = ((D + VW - 1) / VW) * VW; // padded head dim of V and O
  // When V is padded (D = 72 -> 80), column D of every V tile is set to 1.0:
  // PV then also yields the row sum of the bf16 P in O's column D, and the
  // softmax need not add up its exponentials.  (Only when O fits one register
  // group of the epilogue, which reads the sum before normalising.)
  static constexpr bool ONES = DPV > D && (D + 15) / 16 <= 5;
  // With QTMEM (head dims up to 80; chosen for items of at least 24 key
  // steps) Q lives in TMEM, in the columns of the tile's O region that O does
  // not use (DPV + DP / 2 <= 128): S = Q K^T is then a TS product that reads
  // only K from shared memory (2 KB per MMA at N = 64 instead of 6 KB), which
  // relieves the shared-memory bandwidth both tiles' S products and PV share.
  // The epilogue warps move each item's Q there from the TMA-loaded shared
  // tiles once the tile's last S of the previous item is done; on short items
  // that hand-over shows at every item boundary, hence the choice.
  static constexpr bool QTM = QTMEM && D <= 80;
  static constexpr int QCOL = DPV;                    // Q columns at TM_O + X * 128 + QCOL
  static_assert(!QTM || DPV + DP / 2 <= 128, "Q beside O in TMEM");
  // Merge mode (the accumulated partial of earlier KV chunks is merged into
  // the result in the epilogue): for head dims up to 80 the epilogue stages
  // the accumulated rows of one tile in shared memory (one 32 x 16 fp32 block
  // per warp and 16-column chunk) -- tile A's while the item runs, tile B's
  // while tile A is merged -- paid for with a shallower K/V ring; larger head
  // dims load them from global memory one chunk ahead.
  static constexpr int NCH = (D + 15) / 16;            // 16-column chunks of O holding data
  static_assert(!MERGE || NCH <= 5, "staged merge only for head dims up to 80");
  // Head dims up to 80 write the output of a tile through per-warp slots, one
  // 32 x 16 block per chunk, and store them once per tile; merge mode first
  // stages the accumulated blocks in the same slots.
  static constexpr bool SLOTS = NCH <= 5;
  static constexpr int ACCS = SLOTS ? 4 * NCH * EPI_BUF : 0;
  static constexpr int VA = DPV / VW;                  // atoms
  static constexpr int VSW = VW * 2;                   // atom row bytes = swizzle span
  static constexpr int VAT = BLOCK_N * VSW;            // bytes of one atom region
  static constexpr int VTILE = VA * VAT;               // bytes of one V tile
  // two staging buffers per epilogue warp (only without the slots: the
  // space goes to the K/V ring), then the row statistics (m, l) of both tiles
  static constexpr int EPI_STG = SLOTS ? 0 : 4 * 2 * EPI_BUF;
  static constexpr int EPI = EPI_STG + 2 * 2 * BLOCK_M * 4;
  static constexpr int BUDGET = SLOTS ? 232448 - 4096 - EPI - ACCS : 204800;   // bytes for Q and the K/V ring
  static constexpr int QB = (4 * QTILE + 4 * (KTILE + VTILE) <= BUDGET) ? 2 : 1;   // Q double buffer if 4 stages fit
  static constexpr int NS_RAW = (BUDGET - 2 * QB * QTILE) / (KTILE + VTILE);
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;   // K/V ring depth
  using Regs = RegSplit<D <= 80 && !MERGE>;            // the setmaxnreg split of this instantiation
  static constexpr int SMEM = 1024 + 2 * QB * QTILE + NS * (KTILE + VTILE) + ACCS + EPI + 1024;   // + barriers
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(DP <= 128 && DPV <= 128, "head dim too large");
  static_assert(NS >= 4, "ring too shallow");
};

// ---------------------------------------------------------------- exp2
// 2^x on the special-function unit (one MUFU op, flush-to-zero).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe (see ex2_poly2 below), for x <= 8: range reduction
// x = j + f with j the nearest integer (adding 1.5 * 2^23 leaves j in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose
// coefficients were fitted for this kernel by a Remez exchange on relative
// error over [-1/2, 1/2] (max relative error 7.5e-5, far below the bf16
// rounding of P); 2^j is added into the exponent field.  x is clamped at -125
// so the result stays a normal number (masked scores give 2^-125, i.e. 0 for
// all purposes).
constexpr float kP0 = 0.9999280571937561f, kP1 = 0.6932609677314758f;
constexpr float kP2 = 0.2426111251115799f, kP3 = 0.0551716685295105f;

// Of every 8 consecutive score pairs, this many take ex2_poly and the rest the
// MUFU, so the two pipes share the exponentials of the softmax.
constexpr int kPolyPairs = 2;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread until the phase
// completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of the given parity to complete.  The thread
// sleeps in the barrier (woken when the phase completes); the wall clock and
// the abort epoch are only consulted after a sleep of ~0.1 ms that ended
// without the phase, so a normal wait costs no global memory traffic.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t epoch, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    if (*reinterpret_cast<volatile unsigned int *>(&g_attn_abort_epoch) == epoch) return false;
    if (globaltimer() - t0 > WAIT_NS) {
      atomicOr(&g_attn_error, 1u << (site & 31));
      atomicExch(&g_attn_abort_epoch, epoch);
      return false;
    }
  }
}

// Non-blocking test of the phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
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
// The waits on the MMA chain (the issuers' operands and buffers, the
// softmax's S) poll the barrier N times before the sleeping wait: a thread
// woken from a suspended wait resumes later than one that polls, and on
// this chain every cycle of that delay is paid by the tensor pipe (measured:
// 5% of the image-DiT ring launch, 8% of the cached-K/V launch, 3-4% at
// head dim 72).  Bounded: after N polls it is mbar_wait.
constexpr int SPIN_ISSUE = 32, SPIN_SOFTMAX = 8;
template <int N>
__device__ __forceinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, uint32_t epoch, int site) {
  for (int i = 0; i < N; ++i)
    if (mbar_test(bar, parity)) return true;
  return mbar_wait(bar, parity, epoch, site);
}

__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1),
        "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// Tiled bulk store shared -> global (out-of-range rows and columns are dropped).
__device__ __forceinline__ void tma_store_5d(const CUtensorMap *map, const void *src, int c0, int c1, int c2, int c3,
                                             int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one committed bulk store may still be reading its shared memory
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// every committed bulk store has finished reading its shared memory
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

#define TMEM_LD16(taddr, r)                                                                              \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),    \
                 "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
                 "=r"(r[14]), "=r"(r[15])                                                               \
               : "r"(taddr))
#define TMEM_ST16(taddr, r)                                                                              \
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), \
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),       \
                 "r"(r[14]), "r"(r[15])                                                                 \
               : "memory")
#define TMEM_ST8(taddr, r)                                                                               \
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"                       \
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),  \
                 "r"(r[7])                                                                              \
               : "memory")
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// and stride byte offsets (LBO, SBO), version 1 for sm_100, swizzle layout
// 2 = 128B, 4 = 64B, 6 = 32B.
// The same descriptor with everything but the start address fixed at compile
// time: only one 32-bit add per MMA operand at issue time.
template <uint32_t LBO, uint32_t SBO, uint32_t LAYOUT>
__device__ __forceinline__ uint64_t sdesc_c(uint32_t saddr) {
  constexpr uint32_t hi = ((SBO >> 4) & 0x3FFFu) | (1u << 14) | (LAYOUT << 29);
  constexpr uint32_t lo_const = ((LBO >> 4) & 0x3FFFu) << 16;
  return ((uint64_t)hi << 32) | (uint64_t)(((saddr >> 4) & 0x3FFFu) | lo_const);
}
__host__ __device__ constexpr uint32_t layout_of(int swizzle_bytes) {
  return swizzle_bytes == 128 ? 2u : (swizzle_bytes == 64 ? 4u : 6u);
}
// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct Params {
  st::Geom g;
  int lo, n_frames;          // selected frames
  int kv0, kv1;              // key range
  int n_chunks;              // KV chunks the key range is cut into (1: one range)
  int cs[65];                // chunk c starts at key cs[c]; cs[n_chunks] = kv1 (host-computed)
  int nst[64];               // 64-key steps of chunk c
  int tail[64];              // keys in the last step of chunk c
  int ring;                  // 1: every query block starts at the chunk holding its first row
  int n_kv;                  // 64-key steps per item (over all chunks)
  int q_blocks;              // ceil(S / 256)
  int tmode;                 // 1: frames addressed as (t % tblk, b*T/tblk + t/tblk)
  float scale_log2, scale;
  void *o;
  float *lse;
  int o_f32;
  // merge mode: the result is merged with an accumulated fp32 partial and its
  // LSE (read per row by the epilogue; o may alias o_acc)
  const float *o_acc;
  const float *lse_acc;
  int n_items;               // work items of the launch
  int reverse;               // 1: items are walked from the last (merge launches)
  uint32_t epoch;
};

// Packed fp32 pair arithmetic (sm_100 f32x2 instructions).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// The polynomial 2^x of ex2_poly on a pair, with packed arithmetic.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 j = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(j, make_float2(-1.0f, -1.0f), x);
  float2 q = ffma2(make_float2(kP3, kP3), f, make_float2(kP2, kP2));
  q = ffma2(q, f, make_float2(kP1, kP1));
  q = ffma2(q, f, make_float2(kP0, kP0));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// KV chunks: the key range [kv0, kv1) is cut into n_chunks chunks, chunk c
// starting at key kv0 + floor(c * (kv1 - kv0) / n_chunks).  An item walks its
// chunks in ring order from a start chunk (the stationary one), each chunk in
// 64-key steps whose last one may be ragged; the running max, row sum and O
// carry over from one chunk to the next, which is the log-sum-exp merge of the
// chunks in unnormalised form.
// The host computes the chunk edges once per launch (a table in the kernel
// parameters), so the walk does no division.
__device__ __forceinline__ int chunk_lo(const Params &p, int c) { return p.cs[c]; }
struct KeyWalk {
  int c, key, end;           // chunk, first key of the step, end of the chunk
  __device__ __forceinline__ void begin(const Params &p, int c0) {
    c = c0;
    key = chunk_lo(p, c0);
    end = chunk_lo(p, c0 + 1);
  }
  __device__ __forceinline__ void next(const Params &p) {
    key += 64;
    if (key >= end) {
      c = c + 1 == p.n_chunks ? 0 : c + 1;
      key = chunk_lo(p, c);
      end = chunk_lo(p, c + 1);
    }
  }
};
// Ring mode (queries and keys are the same sequence): a query block starts at
// the chunk that holds its first row, as a ring rank starts with its own KV
// chunk before the others arrive.  Otherwise every item starts at chunk 0.
__device__ __forceinline__ int start_chunk(const Params &p, int q0) {
  if (!p.ring) return 0;
  // a first guess, then corrected against the edges; 32-bit arithmetic since
  // q0 * n_chunks < S * n_chunks < 2^32 (the host checks it)
  int c = int((uint32_t(q0) * uint32_t(p.n_chunks)) / uint32_t(p.kv1 - p.kv0));
  while (c + 1 < p.n_chunks && chunk_lo(p, c + 1) <= q0) ++c;
  while (c > 0 && chunk_lo(p, c) > q0) --c;
  return c;
}

// Work item -> (q block, head, frame); q block fastest so that the CTAs that
// run together share K/V tiles in L2.
struct Item {
  int qb, h, t, b, q0, n_qt, c3, c4;
};
__device__ __forceinline__ Item decode(const Params &p, int x) {
  Item it;
  // A merge launch walks the items from the last: the accumulated rows the
  // previous launch wrote last, and the Q tiles it read last, are still in L2
  // when this launch starts.  Every role decodes through here, so all agree.
  if (p.reverse) x = p.n_items - 1 - x;
  it.qb = x % p.q_blocks;
  x /= p.q_blocks;
  it.h = x % p.g.H;
  x /= p.g.H;
  it.t = p.lo + x % p.n_frames;
  it.b = x / p.n_frames;
  it.q0 = it.qb * 2 * BLOCK_M;
  it.n_qt = (p.g.S - it.q0) > BLOCK_M ? 2 : 1;
  if (p.tmode) {
    it.c3 = it.t % p.g.tblk;
    it.c4 = it.b * (p.g.T / p.g.tblk) + it.t / p.g.tblk;
  } else {
    it.c3 = it.t;
    it.c4 = it.b;
  }
  return it;
}

// RING: 0 = one key range; 1 = KV chunks walked in ring order (KeyWalk, the
// last step of a chunk may be ragged); 2 = the same walk when every chunk is a
// whole number of 64-key steps: a rotation of the one-range walk with no
// ragged step, so the softmax needs no key bookkeeping at all.
template <int D, bool MERGE, int RING, bool QTMEM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                   const __grid_constant__ CUtensorMap tk0, const __grid_constant__ CUtensorMap tk1,
                   const __grid_constant__ CUtensorMap tv0, const __grid_constant__ CUtensorMap tv1,
                   const __grid_constant__ CUtensorMap to, const __grid_constant__ CUtensorMap tacc,
                   const __grid_constant__ Params p) {
  using K = Cfg<D, MERGE, QTMEM>;
  constexpr int NS = K::NS, QB = K::QB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                          // QB x 2 Q tiles
  uint8_t *sK = sQ + QB * 2 * K::QTILE;        // NS K tiles
  uint8_t *sV = sK + NS * K::KTILE;            // NS V tiles
  uint8_t *sAcc = sV + NS * K::VTILE;          // merge mode: [epilogue warp][chunk] 32 x 16 fp32 blocks
  uint8_t *sEpi = sAcc + K::ACCS;              // 4 warps x 2 staging buffers (without the slots)
  float *sStat = reinterpret_cast<float *>(sEpi + K::EPI_STG);   // [tile][m | l][row]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + K::EPI);
  uint64_t *q_full = bars;                     // QB
  uint64_t *q_empty = q_full + QB;             // QB, 2 arrivals (the two S issuers)
  uint64_t *k_full = q_empty + QB;             // NS
  uint64_t *k_empty = k_full + NS;             // NS, 2 arrivals (the two S issuers)
  uint64_t *v_full = k_empty + NS;             // NS
  uint64_t *v_empty = v_full + NS;             // NS, 2 arrivals (the two PV issuers)
  // Per (tile X, S buffer b) at index 2X + b.  With two buffers one side can
  // run a step ahead of the other; per-buffer barriers keep every parity wait
  // within one phase.
  uint64_t *s_full = v_empty + NS;             // 4
  uint64_t *p_full = s_full + 4;               // 4, 128 arrivals (softmax threads)
  uint64_t *pv_done = p_full + 4;              // 4
  uint64_t *o_full = pv_done + 4;              // 2
  uint64_t *o_empty = o_full + 2;              // 2, 128 arrivals
  uint64_t *mma_done = o_empty + 2;            // 4, one per issuer
  uint64_t *stat_full = mma_done + 4;          // 2, 128 arrivals (softmax threads)
  uint64_t *stat_empty = stat_full + 2;        // 2, 128 arrivals (epilogue threads)
  uint64_t *v_ready = stat_empty + 2;          // NS: ones column written into the V stage
  uint64_t *acc_full = v_ready + NS;           // [epilogue warp][tile]: the item's accumulated rows landed
  // Q in TMEM (head dims up to 80), per tile: every S of the item done (its Q
  // columns may take the next item's Q), Q of the item in TMEM (128 arrivals
  // of the epilogue threads that moved it)
  uint64_t *s_done = acc_full + 8;             // 2
  uint64_t *qt_full = s_done + 2;              // 2
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(qt_full + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const st::Geom &g = p.g;
  const int n_items = p.q_blocks * g.H * p.n_frames * g.B;
  // one key range: ceil((kv1 - kv0) / 64) steps; ring mode: the steps of every chunk
  const int n_kv = RING ? p.n_kv : (p.kv1 - p.kv0 + BLOCK_N - 1) / BLOCK_N;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, K::QTM ? BLOCK_M : 2);   // with Q in TMEM: the epilogue threads that moved it
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 2);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 2);
      mbar_init(v_ready + i, 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, BLOCK_M);
      mbar_init(pv_done + i, 1);
      mbar_init(mma_done + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, BLOCK_M);
      mbar_init(stat_full + i, BLOCK_M);
      mbar_init(stat_empty + i, BLOCK_M);
    }
    for (int i = 0; i < 8; ++i) mbar_init(acc_full + i, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_done + i, 1);
      mbar_init(qt_full + i, BLOCK_M);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_S0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t epoch = p.epoch;
  // barriers and TMEM are set up: let the next kernel of the stream be
  // scheduled, then wait for the previous one before any global access
  pdl_trigger();
  pdl_wait();

  if (warp >= W_LOAD) {
    // warpgroups 3 and 4: TMA producer, MMA issuers, idle warps
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(K::Regs::ISSUE));
    if (warp == W_LOAD) {
      if (lane == 0 && n_kv > 0) {
        // ================= TMA producer =================
        bool ok = true;
        uint32_t kv = 0;                              // K/V ring position over all items
        int c = 0;                                    // items handled by this CTA
        int last_kv = -1;                             // ring position of the last K/V issued
        for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x, ++c) {
          const Item it = decode(p, x);
          const int qb = c % QB;
          if (!(ok = mbar_wait(q_empty + qb, ((c / QB) & 1) ^ 1, epoch, 0))) break;
          mbar_expect_tx(q_full + qb, it.n_qt * K::QTILE);
          for (int X = 0; X < it.n_qt; ++X) {
            uint8_t *dst = sQ + (qb * 2 + X) * K::QTILE;
            tma_load_5d(dst, &tq0, q_full + qb, 0, it.h, it.q0 + X * BLOCK_M, it.c3, it.c4);
            if (K::C1) tma_load_5d(dst + K::QT0, &tq1, q_full + qb, 64, it.h, it.q0 + X * BLOCK_M, it.c3, it.c4);
          }
          KeyWalk kw;
          if constexpr (RING == 1) kw.begin(p, start_chunk(p, it.q0));
          int rot = 0;                                  // RING == 2: the step's index in the one-range walk
          if constexpr (RING == 2) rot = (chunk_lo(p, start_chunk(p, it.q0)) - p.kv0) / BLOCK_N;
          for (int j = 0; j < n_kv; ++j, ++kv) {
            const int st = kv % NS;
            const uint32_t ph = (kv / NS) & 1;
            const int key = RING == 1 ? kw.key : p.kv0 + (RING == 2 ? rot : j) * BLOCK_N;
            if constexpr (RING == 1) kw.next(p);
            if constexpr (RING == 2) rot = rot + 1 == n_kv ? 0 : rot + 1;
            if (!(ok = mbar_wait(k_empty + st, ph ^ 1, epoch, 1))) break;
            mbar_expect_tx(k_full + st, K::KTILE);
            uint8_t *dk = sK + st * K::KTILE;
            tma_load_5d(dk, &tk0, k_full + st, 0, it.h, key, it.c3, it.c4);
            if (K::C1) tma_load_5d(dk + K::KT0, &tk1, k_full + st, 64, it.h, key, it.c3, it.c4);
            if (!(ok = mbar_wait(v_empty + st, ph ^ 1, epoch, 2))) break;
            mbar_expect_tx(v_full + st, K::VTILE);
            uint8_t *dv = sV + st * K::VTILE;
  #pragma unroll
            for (int a = 0; a < K::VA; ++a)
              tma_load_5d(dv + a * K::VAT, &tv0, v_full + st, a * K::VW, it.h, key, it.c3, it.c4);
            last_kv = (int)kv;
          }
        }
        if (!ok) {
          // drain (bounded, ignoring the abort epoch): the last load issued into every slot
          const unsigned long long t0 = globaltimer();
          for (int i = (last_kv - NS + 1 > 0 ? last_kv - NS + 1 : 0); i <= last_kv; ++i) {
            const uint32_t ph = (i / NS) & 1;
            while (!mbar_try_wait(k_full + i % NS, ph) && globaltimer() - t0 < WAIT_NS) {
            }
            while (!mbar_try_wait(v_full + i % NS, ph) && globaltimer() - t0 < WAIT_NS) {
            }
          }
          for (int i = (c - QB + 1 > 0 ? c - QB + 1 : 0); i <= c && i >= 0; ++i) {
            while (!mbar_try_wait(q_full + i % QB, (i / QB) & 1) && globaltimer() - t0 < WAIT_NS) {
            }
          }
        }
      }
      __syncwarp();
    } else if ((warp == W_S0 || warp == W_S0 + 1) && lane == 0 && n_kv > 0) {
      // ================= S issuer of tile X: S(X, step) = Q_X K^T =================
      const int X = warp - W_S0;
      constexpr uint32_t IDS = idesc_bf16(BLOCK_M, BLOCK_N, 0, 0);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
      bool ok = true;
      uint32_t kv = 0, step = 0;                       // K ring position, S steps of this tile
      int c = 0;
      for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x, ++c) {
        const Item it = decode(p, x);
        const int qb = c % QB;
        // the item's Q: in shared memory, or (head dims up to 80) moved into TMEM by the epilogue
        if (!(ok = K::QTM ? mbar_wait(qt_full + X, c & 1, epoch, 3) : mbar_wait(q_full + qb, (c / QB) & 1, epoch, 3)))
          break;
        if (X >= it.n_qt) {
          // tile absent from this item: release the shared K stages and Q in step
          for (int j = 0; j < n_kv && ok; ++j) {
            const uint32_t g0 = kv + j;
            if (!(ok = mbar_wait(k_full + g0 % NS, (g0 / NS) & 1, epoch, 4))) break;
            mbar_arrive(k_empty + g0 % NS);
          }
          if (!ok) break;
          if (K::QTM) mbar_arrive(s_done + X);
          else mbar_arrive(q_empty + qb);
          kv += n_kv;
          continue;
        }
        const uint32_t qa = aQ + (qb * 2 + X) * K::QTILE;
        const uint32_t qt = tmem + TM_O + X * 128 + K::QCOL;   // Q in TMEM: K-slice kk at columns 8 kk
        for (int j = 0; j < n_kv && ok; ++j, ++step) {
          const uint32_t g0 = kv + j;
          const int st = g0 % NS;
          const uint32_t b = step & 1;
          // S(step) overwrites P(step - 2) in the same buffer: PV(step - 2) must be done
          if (step >= 2 && !(ok = mbar_wait_spin<SPIN_ISSUE>(pv_done + 2 * X + b, ((step - 2) >> 1) & 1, epoch, 5))) break;
          if (!(ok = mbar_wait_spin<SPIN_ISSUE>(k_full + st, (g0 / NS) & 1, epoch, 4))) break;
          tc_fence_after();
          const uint32_t d = tmem + X * 2 * BLOCK_N + b * BLOCK_N;
          const uint32_t ka = aK + st * K::KTILE;
  #pragma unroll
          for (int kk = 0; kk < K::C0 / 16; ++kk) {
            if constexpr (K::QTM)
              mma_ts(d, qt + kk * 8, sdesc_c<16, 8 * K::SW0, layout_of(K::SW0)>(ka + kk * 32), IDS, kk > 0);
            else
              mma_ss(d, sdesc_c<16, 8 * K::SW0, layout_of(K::SW0)>(qa + kk * 32),
                     sdesc_c<16, 8 * K::SW0, layout_of(K::SW0)>(ka + kk * 32), IDS, kk > 0);
          }
          if (K::C1) {
  #pragma unroll
            for (int kk = 0; kk < (K::C1 ? K::C1 : 16) / 16; ++kk) {
              if constexpr (K::QTM)
                mma_ts(d, qt + K::C0 / 2 + kk * 8,
                       sdesc_c<16, 8 * (K::SW1 ? K::SW1 : 32), layout_of(K::SW1 ? K::SW1 : 32)>(ka + K::KT0 + kk * 32),
                       IDS, 1);
              else
                mma_ss(d, sdesc_c<16, 8 * (K::SW1 ? K::SW1 : 32), layout_of(K::SW1 ? K::SW1 : 32)>(qa + K::QT0 + kk * 32),
                       sdesc_c<16, 8 * (K::SW1 ? K::SW1 : 32), layout_of(K::SW1 ? K::SW1 : 32)>(ka + K::KT0 + kk * 32),
                       IDS, 1);
            }
          }
          tc_commit(s_full + 2 * X + b);
          tc_commit(k_empty + st);
          // last S of this item issued: its Q (shared tiles, or the TMEM columns) may be replaced
          if (j + 1 == n_kv) tc_commit(K::QTM ? s_done + X : q_empty + qb);
        }
        kv += n_kv;
      }
      // every MMA issued by this thread completes before TMEM is released
      tc_commit(mma_done + warp - W_S0);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(mma_done + warp - W_S0, 0) && globaltimer() - t0 < WAIT_NS) {
      }
    } else if ((warp == W_PV0 || warp == W_PV0 + 1) && lane == 0 && n_kv > 0) {
      // ================= PV issuer of tile X: O_X += P(X, step) V =================
      const int X = warp - W_PV0;
      constexpr uint32_t IDPV = idesc_bf16(BLOCK_M, K::DPV, 0, 1);
      const uint32_t aV = smem_u32(sV);
      bool ok = true;
      uint32_t kv = 0, step = 0, oc = 0;
      for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x) {
        const Item it = decode(p, x);
        if (X >= it.n_qt) {
          // tile absent from this item: release the shared V stages in step
          for (int j = 0; j < n_kv && ok; ++j) {
            const uint32_t g0 = kv + j;
            if (!(ok = mbar_wait(v_full + g0 % NS, (g0 / NS) & 1, epoch, 6))) break;
            mbar_arrive(v_empty + g0 % NS);
          }
          kv += n_kv;
          continue;
        }
        for (int j = 0; j < n_kv && ok; ++j, ++step) {
          const uint32_t g0 = kv + j;
          const int st = g0 % NS;
          const uint32_t b = step & 1;
          if (!(ok = mbar_wait_spin<SPIN_ISSUE>((K::ONES ? v_ready : v_full) + st, (g0 / NS) & 1, epoch, 6))) break;
          if (!(ok = mbar_wait_spin<SPIN_ISSUE>(p_full + 2 * X + b, (step >> 1) & 1, epoch, 7 + X))) break;
          // O of the tile's previous item read out by the epilogue
          if (j == 0 && !(ok = mbar_wait(o_empty + X, (oc & 1) ^ 1u, epoch, 9 + X))) break;
          tc_fence_after();
          const uint32_t d = tmem + TM_O + X * 128;
          const uint32_t pa = tmem + X * 2 * BLOCK_N + b * BLOCK_N;   // P (bf16 pairs) over the S columns
          const uint32_t va = aV + st * K::VTILE;
  #pragma unroll
          for (int kk = 0; kk < BLOCK_N / 16; ++kk)
            mma_ts(d, pa + kk * 8, sdesc_c<K::VAT, 8 * K::VSW, layout_of(K::VSW)>(va + kk * 16 * K::VSW), IDPV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(pv_done + 2 * X + b);
          tc_commit(v_empty + st);
        }
        if (!ok) break;
        tc_commit(o_full + X);
        ++oc;
        kv += n_kv;
      }
      tc_commit(mma_done + 2 + X);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(mma_done + 2 + X, 0) && globaltimer() - t0 < WAIT_NS) {
      }
    } else if (K::ONES && warp == W_ONES && n_kv > 0) {
      // ================= ones column of every V stage =================
      // Column D lies in atom D / VW at element D % VW of each 64-key row;
      // the row's 16-byte chunks are permuted by the atom's swizzle.
      constexpr int A1 = D / K::VW, XB = (D % K::VW) * 2;
      constexpr int CHK = XB >> 4, WITHIN = XB & 15;
      bool ok = true;
      uint32_t kv = 0;
      for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x) {
        for (int j = 0; j < n_kv; ++j, ++kv) {
          const int st = kv % NS;
          if (lane == 0) ok = mbar_wait(v_full + st, (kv / NS) & 1, epoch, 21);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          __syncwarp();                        // the copy's zero fill of the column is done
          uint8_t *vt = sV + st * K::VTILE + A1 * K::VAT;
          for (int r = lane; r < BLOCK_N; r += 32) {
            const int sw = K::VSW == 128 ? (r & 7) : (K::VSW == 64 ? ((r >> 1) & 3) : ((r >> 2) & 1));
            *reinterpret_cast<uint16_t *>(vt + r * K::VSW + ((CHK ^ sw) << 4) + WITHIN) = 0x3F80;   // bf16 1.0
          }
          fence_async_smem();                  // visible to the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(v_ready + st);
        }
      }
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(K::Regs::SOFTMAX));
    // ================= softmax warpgroups =================
    const int X = warp >> 2;                   // tile
    const int r = ((warp & 3) << 5) + lane;    // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + X * 2 * BLOCK_N;
    const uint32_t tO = tmem + lane_off + TM_O + X * 128;
    const float sl2 = p.scale_log2;
    const float2 scale2 = make_float2(sl2, sl2);
    uint32_t gs = 0, oc = 0;                   // S steps and items of this tile
    bool ok = n_kv > 0;                        // an empty key range is written by the epilogue alone
    for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x) {
      const Item it = decode(p, x);
      if (X >= it.n_qt) continue;
      float m = -INFINITY, l = 0.f;
      // RING == 1: the chunk whose last (possibly ragged) step comes next, and
      // that step's index in the item's walk
      int rc = 0, jr = 0;
      if constexpr (RING == 1) {
        rc = start_chunk(p, it.q0);
        jr = p.nst[rc] - 1;
      }
      for (int j = 0; j < n_kv; ++j, ++gs) {
        const uint32_t b = gs & 1;
        if (!(ok = mbar_wait_spin<SPIN_SOFTMAX>(s_full + 2 * X + b, (gs >> 1) & 1, epoch, 11 + X))) break;
        tc_fence_after();
        uint32_t sr[BLOCK_N];
#pragma unroll
        for (int c = 0; c < BLOCK_N / 16; ++c) TMEM_LD16(tS + b * BLOCK_N + c * 16, (sr + c * 16));
        tmem_wait_ld();
        int nvalid = BLOCK_N;
        if constexpr (RING == 1) {
          if (j == jr) {                       // a chunk's last step: mask past its end, go to the next chunk
            nvalid = p.tail[rc];
            rc = rc + 1 == p.n_chunks ? 0 : rc + 1;
            jr += p.nst[rc];
          }
        } else if constexpr (RING == 0) {
          nvalid = p.kv1 - (p.kv0 + j * BLOCK_N);
        }
        if (nvalid < BLOCK_N) {
#pragma unroll
          for (int c = 0; c < BLOCK_N; ++c)
            if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
        }
        float mxp[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mxp[e] = __uint_as_float(sr[e]);
#pragma unroll
        for (int c = 4; c < BLOCK_N; c += 8) {
          mxp[0] = fmax3(mxp[0], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          mxp[1] = fmax3(mxp[1], __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          if (c + 4 < BLOCK_N) {
            mxp[2] = fmax3(mxp[2], __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
            mxp[3] = fmax3(mxp[3], __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
          }
        }
        const float mx = fmaxf(fmax3(mxp[0], mxp[1], mxp[2]), mxp[3]) * sl2;
        if (j == 0) {
          m = mx;
        } else {
          const bool need = mx > m + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // O holds PV up to step gs-1: wait for it, then rescale in TMEM
            if (!(ok = mbar_wait(pv_done + 2 * X + ((gs - 1) & 1), ((gs - 1) >> 1) & 1, epoch, 15 + X))) break;
            tc_fence_after();
            const float corr = need ? ex2_mufu(m - mx) : 1.0f;
            if (need) {
              if (!K::ONES) l *= corr;         // with the ones column the sum is rescaled with O
              m = mx;
            }
#pragma unroll 1
            for (int c = 0; c < K::DPV / 16; ++c) {
              uint32_t ov[16];
              TMEM_LD16(tO + c * 16, ov);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
              TMEM_ST16(tO + c * 16, ov);
            }
            tmem_wait_st();
          }
        }
        const float2 negm = make_float2(-m, -m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int c0 = 0; c0 < BLOCK_N; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 xx = ffma2(make_float2(__uint_as_float(sr[c0 + c]), __uint_as_float(sr[c0 + c + 1])),
                                    scale2, negm);
            float2 e;
            if (((c >> 1) & 7) < kPolyPairs) {
              e = ex2_poly2(xx);
            } else {
              e.x = ex2_mufu(xx.x);
              e.y = ex2_mufu(xx.y);
            }
            if (!K::ONES) acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], e);
            pk[c >> 1] = st::pack_bf16x2(e.x, e.y);
          }
          TMEM_ST16(tS + b * BLOCK_N + (c0 >> 1), pk);
        }
        if (!K::ONES) {
          const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
          const float2 a = fadd2(a01, a23);
          l += a.x + a.y;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + 2 * X + b);
      }
      if (!ok) break;
      // hand the row statistics to the epilogue warpgroup
      if (!(ok = mbar_wait(stat_empty + X, (oc & 1) ^ 1, epoch, 13 + X))) break;
      sStat[(X * 2 + 0) * BLOCK_M + r] = m;
      sStat[(X * 2 + 1) * BLOCK_M + r] = l;
      mbar_arrive(stat_full + X);
      ++oc;
    }
  } else {
    // the epilogue keeps the launch's 96 registers in the wide split
    if constexpr (K::Regs::EPI > 96) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(K::Regs::EPI));
    // ================= epilogue warpgroup =================
    // Per tile: wait for the last PV and the row statistics, read O out of
    // TMEM into registers (TMEM is released right after), divide by the row
    // sum, stage each 32 x 16 block of this warp in shared memory in the
    // swizzled layout of the output tensor map, and let one lane write it
    // with a bulk tensor store (rows past S and columns past D are dropped by
    // the copy engine).  The LSE is written per row.
    const int qd = warp - W_EPI;               // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    uint8_t *stg = sEpi + qd * 2 * EPI_BUF;
    uint32_t oc0 = 0, oc1 = 0, nst = 0;        // items per tile, bulk stores issued by this warp
    bool ok = true;
    bool acc_pending[2] = {false, false};      // merge mode: staged loads issued and not yet waited for
    uint32_t acc_par[2] = {0u, 0u};            // ... and the barrier phase they complete
    // the copy engine brings the accumulated rows of tile XX of the current
    // item (this warp's 32 rows, every chunk) into this warp's staging area
#define STAGE_ACC(XX, ROW0)                                                                                  \
  {                                                                                                          \
    __syncwarp(); /* the area's previous contents are read */                                                \
    if (lane == 0) {                                                                                         \
      bulk_wait_read0(); /* ... also by the stores of merged blocks that went out from it */                 \
      fence_async_smem(); /* ... and ordered before the copies that overwrite them */                        \
      mbar_expect_tx(acc_full + qd * 2 + (XX), K::NCH * EPI_BUF);                                            \
      _Pragma("unroll") for (int k = 0; k < K::NCH; ++k)                                                     \
        tma_load_5d(sAcc + (qd * K::NCH + k) * EPI_BUF, &tacc, acc_full + qd * 2 + (XX), k * EPI_COLS, it.h, \
                    (ROW0), it.c3, it.c4);                                                                   \
    }                                                                                                        \
    acc_pending[XX] = true;                                                                                  \
    acc_par[XX] = ((XX) ? oc1 : oc0) & 1; /* items of the tile so far = the phase of these copies */        \
  }
    // Q in TMEM (head dims up to 80): the epilogue warps move each item's Q
    // rows (lane = row, this warp's quadrant of 32 rows) from the swizzled
    // shared tiles the TMA loaded into the tile's Q columns beside O -- for
    // item c + 1 as soon as the tile's last S of item c is done, before item
    // c's O is read out -- and then release the shared tiles to the loader.
    auto move_q = [&](int c) -> bool {
      const int qb = c % QB;
      if (!mbar_wait(q_full + qb, (c / QB) & 1, epoch, 24)) return false;
      const int row = qd * 32 + lane;
      for (int X = 0; X < 2; ++X) {
        if (c > 0 && !mbar_wait(s_done + X, (c - 1) & 1, epoch, 25 + X)) return false;
        tc_fence_after();
        const uint8_t *tile = sQ + (qb * 2 + X) * K::QTILE;
        const uint32_t tq = tmem + lane_off + TM_O + X * 128 + K::QCOL;
        // the 16-byte chunks of one row of a part, un-swizzled: 128-byte rows
        // swizzle chunk f to f ^ (r & 7), 64-byte rows to f ^ ((r >> 1) & 3),
        // 32-byte rows to f ^ ((r >> 2) & 1); every 16 bytes are 4 columns
        auto part = [&](const uint8_t *base, int row_bytes, uint32_t col) {
          const uint8_t *src = base + row * row_bytes;
          const int sw = row_bytes == 128 ? (row & 7) : (row_bytes == 64 ? ((row >> 1) & 3) : ((row >> 2) & 1));
          for (int f0 = 0; f0 < row_bytes / 16; f0 += 4) {
            uint32_t v[16];
            const int nf = row_bytes / 16 - f0 < 4 ? row_bytes / 16 - f0 : 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (i < nf) {
                const uint4 w = *reinterpret_cast<const uint4 *>(src + (((f0 + i) ^ sw) << 4));
                v[4 * i] = w.x;
                v[4 * i + 1] = w.y;
                v[4 * i + 2] = w.z;
                v[4 * i + 3] = w.w;
              }
            }
            if (nf == 4) TMEM_ST16(tq + col + f0 * 4, v);
            else TMEM_ST8(tq + col + f0 * 4, v);            // a 32-byte part: 8 columns
          }
        };
        part(tile, K::SW0, 0);
        if (K::C1) part(tile + K::QT0, K::SW1 ? K::SW1 : 32, K::C0 / 2);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(qt_full + X);
      }
      mbar_arrive(q_empty + qb);
      return true;
    };
    if (K::QTM && n_kv > 0 && (int)blockIdx.x < n_items) ok = move_q(0);
    int citem = 0;                             // items of this CTA so far
    for (int x = blockIdx.x; x < n_items && ok; x += gridDim.x, ++citem) {
      const Item it = decode(p, x);
      float la_t[2] = {-INFINITY, -INFINITY};  // merge mode: accumulated LSE of this lane's row per tile
      if ((MERGE || K::NCH > 5) && p.o_acc && n_kv > 0) {
        // the accumulated rows this warp merges at the end of the item: with a
        // staging area the copy engine brings them into shared memory now,
        // otherwise into L2, while the item's steps run
        for (int X = 0; X < it.n_qt; ++X) {
          const int row0 = it.q0 + X * BLOCK_M + qd * 32;
          const int qrow = row0 + lane;
          if (qrow < g.S) la_t[X] = p.lse_acc[(((long long)it.b * g.T + it.t) * g.H + it.h) * g.S + qrow];
          if (MERGE && X == 0) {
            STAGE_ACC(0, row0);                // tile B's rows follow once tile A is merged
          } else if (qrow < g.S) {
            const float *src = p.o_acc + g.frame(it.b, it.t) + g.token(qrow) + (long long)it.h * D;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(uint32_t(D * 4)) : "memory");
          }
        }
      }
      // the next item's Q goes into TMEM once this item's S products are done
      // (after the accumulated rows above were requested, so those copies run
      // during this item's steps)
      if (K::QTM && n_kv > 0 && x + (int)gridDim.x < n_items && !(ok = move_q(citem + 1))) break;
      for (int X = 0; X < it.n_qt && ok; ++X) {
        const int r = qd * 32 + lane;
        const int qrow = it.q0 + X * BLOCK_M + r;
        const bool valid = qrow < g.S;
        const long long lse_idx = (((long long)it.b * g.T + it.t) * g.H + it.h) * g.S + qrow;
        if (n_kv == 0) {
          // empty key range: o = 0, lse = -inf (merged: the accumulated result unchanged)
          if (valid) {
            const long long off = g.frame(it.b, it.t) + g.token(qrow) + (long long)it.h * D;
            const bool acc = p.o_acc && p.lse_acc[lse_idx] != -INFINITY;
            for (int d = 0; d < D; ++d) {
              const float x = acc ? p.o_acc[off + d] : 0.f;
              if (p.o_f32) static_cast<float *>(p.o)[off + d] = x;
              else static_cast<uint16_t *>(p.o)[off + d] = st::f32_to_bf16(x);
            }
            if (p.lse) p.lse[lse_idx] = p.lse_acc ? p.lse_acc[lse_idx] : -INFINITY;
          }
          continue;
        }
        const uint32_t ocx = X ? oc1 : oc0;
        const long long off = valid ? g.frame(it.b, it.t) + g.token(qrow) + (long long)it.h * D : 0;
        // merge flow: the accumulated LSE of the row was loaded at the start of
        // the item; the accumulated partial is read from the staging area
        // (MERGE) or from global memory one 16-column chunk ahead of its use
        // (head dims up to 80 merge only in the MERGE instantiation)
        const bool merging = (MERGE || K::NCH > 5) && p.o_acc != nullptr;
        const float la = la_t[X];
        const bool use_acc = la != -INFINITY;  // nothing accumulated: the partial is not read
        const float *arow = p.o_acc + off;
        float4 an[4];                          // accumulated chunk, one ahead (global flow)
#define ST_LOAD_ACC(k)                                                                                       \
  _Pragma("unroll") for (int f = 0; f < 4; ++f) {                                                            \
    an[f] = make_float4(0.f, 0.f, 0.f, 0.f);                                                                 \
    if (valid && (k) * 16 + 4 * f < D) an[f] = *reinterpret_cast<const float4 *>(arow + (k) * 16 + 4 * f);   \
  }
        if (!MERGE && merging) { ST_LOAD_ACC(0) }
        if (!(ok = mbar_wait(o_full + X, ocx & 1, epoch, 17 + X))) break;
        if (!(ok = mbar_wait(stat_full + X, ocx & 1, epoch, 19 + X))) break;
        if (X) ++oc1;
        else ++oc0;
        tc_fence_after();
        const float m = sStat[(X * 2 + 0) * BLOCK_M + r];
        float l = sStat[(X * 2 + 1) * BLOCK_M + r];   // replaced by O's column D with the ones column
        mbar_arrive(stat_empty + X);
        float inv = 1.0f / l;
        float fa = 0.f, lse_row = 0.f;         // weight of the accumulated partial; LSE of the row
        const uint32_t tO = tmem + lane_off + TM_O + X * 128;
        constexpr int NCH = (D + EPI_COLS - 1) / EPI_COLS;    // 16-column chunks holding data
        constexpr int G0 = NCH > 5 ? 4 : NCH;                  // chunks of the first register group
        // O leaves TMEM in at most two register groups; TMEM is released as
        // soon as the last group is loaded, before anything is stored.
#pragma unroll
        for (int grp = 0; grp < (NCH > G0 ? 2 : 1); ++grp) {
          const int c0 = grp * G0;
          const int nch = grp == 0 ? G0 : NCH - G0;
          uint32_t ov[G0][16];
#pragma unroll
          for (int c = 0; c < G0; ++c)
            if (c < nch) TMEM_LD16(tO + (c0 + c) * 16, ov[c]);
          tmem_wait_ld();
          if (K::ONES && grp == 0) {           // row sum of the bf16 P, accumulated by PV
            l = __uint_as_float(ov[D / 16][D % 16]);
            inv = 1.0f / l;
          }
          if (grp == 0) {
            // this chunk's natural-log LSE; merged with the accumulated one when asked:
            //   w_a = exp(lse_a - M), w_c = exp(lse_c - M), o = (w_a o_a + w_c O / l) / (w_a + w_c)
            lse_row = (m + log2f(l)) * 0.6931471805599453f;
            if (merging) {
              const float M = fmaxf(la, lse_row);
              const float wa = expf(la - M), wc = expf(lse_row - M);
              const float sw = wa + wc;
              fa = wa / sw;
              inv = wc / (sw * l);
              lse_row = M + logf(sw);
            }
          }
          if (c0 + nch == NCH) {
            tc_fence_before();
            mbar_arrive(o_empty + X);          // O of this tile may be overwritten
          }
          const int row0 = it.q0 + X * BLOCK_M + qd * 32;
          {
#pragma unroll
          for (int c = 0; c < G0; ++c, ++nst) {
            if (c >= nch) break;
            uint8_t *buf = stg + (nst & 1) * EPI_BUF;
            float *y = reinterpret_cast<float *>(ov[c]);
            if (merging) {
              // o = fa * o_acc + O * inv, with fa = w_a / (w_a + w_c), inv = w_c / ((w_a + w_c) l)
              float a[16];
              if constexpr (MERGE) {
                if (c0 + c == 0) {             // the item's staged rows of this warp and tile have landed
                  bool got = true;
                  if (lane == 0) got = mbar_wait(acc_full + qd * 2 + X, ocx & 1, epoch, 23);
                  if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
                    ok = false;
                    break;
                  }
                  acc_pending[X] = false;
                  __syncwarp();
                }
                // 64B swizzle of the fp32 block: 16-byte chunk f of row r at f ^ ((r >> 1) & 3)
                const uint8_t *ab = sAcc + (qd * K::NCH + c0 + c) * EPI_BUF + lane * 64;
#pragma unroll
                for (int f = 0; f < 4; ++f) an[f] = *reinterpret_cast<const float4 *>(ab + ((f ^ ((lane >> 1) & 3)) << 4));
              }
#pragma unroll
              for (int f = 0; f < 4; ++f) {   // a row with nothing accumulated is not used (may hold NaN)
                a[4 * f] = use_acc ? an[f].x : 0.f;
                a[4 * f + 1] = use_acc ? an[f].y : 0.f;
                a[4 * f + 2] = use_acc ? an[f].z : 0.f;
                a[4 * f + 3] = use_acc ? an[f].w : 0.f;
              }
              if (!MERGE && c0 + c + 1 < NCH) { ST_LOAD_ACC(c0 + c + 1) }
#pragma unroll
              for (int e = 0; e < 16; ++e) y[e] = fmaf(fa, a[e], __uint_as_float(ov[c][e]) * inv);
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) y[e] = __uint_as_float(ov[c][e]) * inv;
            }
            if constexpr (K::SLOTS) {
              // the block goes out from its slot (merge mode: the slot its
              // accumulated block came from, which every lane has read), one
              // store per block once the tile's blocks are all written; the
              // stores of the previous tile must have read the slots
              if (!MERGE && c0 + c == 0 && lane == 0) bulk_wait_read0();
              buf = sAcc + (qd * K::NCH + c0 + c) * EPI_BUF;
              __syncwarp();
            } else {
              if (lane == 0) bulk_wait_read1();  // the store that used this buffer has read it
              __syncwarp();
            }
            if (p.o_f32) {
              // 64-byte rows, 64B swizzle: 16-byte chunk f of row r at f ^ ((r >> 1) & 3)
#pragma unroll
              for (int f = 0; f < 4; ++f)
                *reinterpret_cast<float4 *>(buf + lane * 64 + ((f ^ ((lane >> 1) & 3)) << 4)) =
                    make_float4(y[4 * f], y[4 * f + 1], y[4 * f + 2], y[4 * f + 3]);
            } else {
              // 32-byte rows, 32B swizzle: 16-byte chunk f of row r at f ^ ((r >> 2) & 1)
#pragma unroll
              for (int f = 0; f < 2; ++f) {
                uint4 w;
                w.x = st::pack_bf16x2(y[8 * f], y[8 * f + 1]);
                w.y = st::pack_bf16x2(y[8 * f + 2], y[8 * f + 3]);
                w.z = st::pack_bf16x2(y[8 * f + 4], y[8 * f + 5]);
                w.w = st::pack_bf16x2(y[8 * f + 6], y[8 * f + 7]);
                *reinterpret_cast<uint4 *>(buf + lane * 32 + ((f ^ ((lane >> 2) & 1)) << 4)) = w;
              }
            }
            if (!K::SLOTS) {
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                // a block wholly past the last row stores nothing, but still
                // commits a (empty) group so the buffer accounting stays in step
                if (row0 < g.S) tma_store_5d(&to, buf, (c0 + c) * EPI_COLS, it.h, row0, it.c3, it.c4);
                bulk_commit();
              }
            }
          }
          if (K::SLOTS && ok) {                // the tile's blocks, one bulk store each
            fence_async_smem();
            __syncwarp();
            if (lane == 0 && row0 < g.S) {
              for (int c = 0; c < nch; ++c)
                tma_store_5d(&to, sAcc + (qd * K::NCH + c0 + c) * EPI_BUF, (c0 + c) * EPI_COLS, it.h, row0,
                             it.c3, it.c4);
              bulk_commit();
            }
          }
          }
        }
#undef ST_LOAD_ACC
        if (!ok) break;
        // tile A is merged: its staging area takes tile B's rows (in L2 since the item started)
        if (MERGE && merging && X == 0 && it.n_qt == 2) STAGE_ACC(1, it.q0 + BLOCK_M + qd * 32)
        if (valid && p.lse) p.lse[lse_idx] = lse_row;
      }
    }
    if (lane == 0) bulk_wait_all();
#undef STAGE_ACC
    if (MERGE && lane == 0) {
      // after an abort: staged copies into this warp's area may still be in
      // flight; wait for them (bounded, ignoring the abort epoch) before exiting
      const unsigned long long t0 = globaltimer();
      for (int X = 0; X < 2; ++X)
        if (acc_pending[X])
          while (!mbar_try_wait(acc_full + qd * 2 + X, acc_par[X]) && globaltimer() - t0 < WAIT_NS) {
          }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_S0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
  }
}

// Trivial kernel used by the failure-detection self test: waits on an
// mbarrier nothing arrives on, with a short limit, through the same bounded
// wait as the attention kernel.
__global__ void wait_timeout_probe(unsigned long long limit_ns, uint32_t epoch) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer() - t0 > limit_ns) {
        atomicOr(&g_attn_error, 1u << 31);
        break;
      }
    }
  }
}

// Evaluates the softmax's two exponentials element by element, for the
// self test of their error: the FMA-pipe polynomial (ex2_poly2) and the MUFU
// instruction (ex2_mufu), exactly as the softmax calls them.
__global__ void ex2_probe(const float *__restrict__ x, float *__restrict__ y_poly, float *__restrict__ y_mufu,
                          int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = x[i];
  const float2 r = ex2_poly2(make_float2(a, a));
  y_poly[i] = r.x;
  y_mufu[i] = ex2_mufu(a);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swz(int bytes) {
  return bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                      : (bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// 5-D map over (d, h, s, frame-in-block, block) with a box of (box_d, 1, box_rows, 1, 1);
// elements are bf16, or fp32 when f32 is set.
bool make_map(CUtensorMap *m, const void *ptr, const st::Geom &g, int tmode, int box_d, int swizzle_bytes,
              int box_rows, int f32 = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es_bytes = f32 ? 4 : 2;
  cuuint64_t dims[5], strides[4];
  dims[0] = (cuuint64_t)g.D;
  dims[1] = (cuuint64_t)g.H;
  dims[2] = (cuuint64_t)g.S;
  strides[0] = (cuuint64_t)g.D * es_bytes;
  strides[1] = (cuuint64_t)g.ss * es_bytes;
  if (tmode) {
    dims[3] = (cuuint64_t)g.tblk;
    dims[4] = (cuuint64_t)g.B * (g.T / g.tblk);
    strides[2] = (cuuint64_t)g.st * es_bytes;
    strides[3] = (cuuint64_t)g.stb * es_bytes;
  } else {
    dims[3] = (cuuint64_t)g.T;
    dims[4] = (cuuint64_t)g.B;
    strides[2] = (cuuint64_t)g.st * es_bytes;
    strides[3] = (cuuint64_t)g.sb * es_bytes;
  }
  cuuint32_t box[5] = {(cuuint32_t)box_d, 1, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                  const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz(swizzle_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

std::atomic<uint32_t> g_epoch{0};

template <int D, bool MERGE, int RING = 0, bool QTMEM = false>
st_status launch_spatial(const st::Geom &g, int lo, int hi, int kv0, int kv1, float scale, const void *q,
                         const void *k, const void *v, void *o, float *lse, int o_f32, cudaStream_t s,
                         const float *o_acc, const float *lse_acc, int n_chunks, int ring) {
  using K = Cfg<D, MERGE, QTMEM>;
  const int tmode = g.tblk != g.T ? 1 : 0;
  CUtensorMap m[8];
  const int c1 = K::C1 ? K::C1 : 16;
  if (!make_map(&m[0], q, g, tmode, K::C0, K::SW0, BLOCK_M) || !make_map(&m[1], q, g, tmode, c1, c1 * 2, BLOCK_M) ||
      !make_map(&m[2], k, g, tmode, K::C0, K::SW0, BLOCK_N) || !make_map(&m[3], k, g, tmode, c1, c1 * 2, BLOCK_N) ||
      !make_map(&m[4], v, g, tmode, K::VW, K::VSW, BLOCK_N) || !make_map(&m[5], v, g, tmode, K::VW, K::VSW, BLOCK_N) ||
      !make_map(&m[6], o, g, tmode, EPI_COLS, EPI_COLS * (o_f32 ? 4 : 2), 32, o_f32))
    return ST_ERR_CUDA;
  // fp32 accumulator blocks staged by the merge mode (unused otherwise)
  if (o_acc) {
    if (!make_map(&m[7], o_acc, g, tmode, EPI_COLS, EPI_COLS * 4, 32, 1)) return ST_ERR_CUDA;
  } else {
    memset(&m[7], 0, sizeof(m[7]));
  }
  Params p;
  p.g = g;
  p.lo = lo;
  p.n_frames = hi - lo;
  p.kv0 = kv0;
  p.kv1 = kv1;
  p.n_chunks = n_chunks;
  p.ring = ring;
  {
    if (n_chunks < 1 || n_chunks > 64) return ST_ERR_SHAPE;
    long long steps = 0;                       // 64-key steps over every chunk
    for (int c = 0; c <= n_chunks; ++c) p.cs[c] = int(kv0 + ((long long)c * (kv1 - kv0)) / n_chunks);
    for (int c = 0; c < n_chunks; ++c) {
      p.nst[c] = (p.cs[c + 1] - p.cs[c] + BLOCK_N - 1) / BLOCK_N;
      p.tail[c] = p.cs[c + 1] - p.cs[c] - (p.nst[c] - 1) * BLOCK_N;
      steps += p.nst[c];
    }
    p.n_kv = int(steps);
  }
  p.q_blocks = (g.S + 2 * BLOCK_M - 1) / (2 * BLOCK_M);
  p.tmode = tmode;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o;
  p.lse = lse;
  p.o_f32 = o_f32;
  p.o_acc = o_acc;
  p.lse_acc = lse_acc;
  p.epoch = g_epoch.fetch_add(1) + 1;
  const long long items = (long long)p.q_blocks * g.H * g.B * p.n_frames;
  if (items <= 0) return ST_OK;
  if (items > 0x7fffffffLL) return ST_ERR_SHAPE;
  p.n_items = int(items);
  p.reverse = o_acc != nullptr ? 1 : 0;
  const int ctas = int(items < st::num_sms() ? items : st::num_sms());  // persistent: one CTA per SM
  auto kern = attn_fwd_sm100<D, MERGE, RING, QTMEM>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM) != cudaSuccess)
    return ST_ERR_CUDA;
  // The register split of the warpgroups (setmaxnreg) assumes the launch
  // grants 96 registers per thread; with fewer, the warpgroups that ask for
  // more would wait forever.  Refuse to launch such a build.
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ST_ERR_CUDA;
    regs_ok = fa.numRegs * NUM_THREADS >= 256 * K::Regs::SOFTMAX + 128 * K::Regs::EPI + 256 * K::Regs::ISSUE ? 1 : 0;
  }
  if (!regs_ok) return ST_ERR_UNSUPPORTED;
  return st::launch_pdl(kern, ctas, NUM_THREADS, K::SMEM, s, m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], p);
}

}  // namespace

namespace st {

unsigned int read_and_clear_attn_error(cudaStream_t stream, cudaError_t *err) {
  unsigned int word = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&word, g_attn_error, sizeof(word), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_attn_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (err) *err = e;
  return word;
}

st_status attn_spatial_sm100(const Geom &g, int lo, int hi, int kv0, int kv1, float scale, const void *q,
                             const void *k, const void *v, void *o, float *lse, int o_f32, cudaStream_t s,
                             const float *o_acc, const float *lse_acc, int n_chunks, int ring) {
  if (hi <= lo) return ST_OK;
  if (n_chunks < 1 || (n_chunks > 1 && n_chunks > kv1 - kv0) || (ring && (kv0 != 0 || kv1 != g.S || o_acc)))
    return ST_ERR_SHAPE;
  if ((long long)(kv1 - kv0) * n_chunks >= (1LL << 32)) return ST_ERR_SHAPE;   // chunk edges in 32 bits
  // 64-key steps per item: head dims 72 and 80 keep Q in TMEM when an item
  // has at least 24 of them (the per-item hand-over of Q costs more than the
  // shared-memory bandwidth it frees on shorter items)
  long long steps = 0;
  bool aligned = true;                         // every chunk a whole number of 64-key steps
  for (int c = 0; c < n_chunks; ++c) {
    const long long a = kv0 + ((long long)c * (kv1 - kv0)) / n_chunks;
    const long long b = kv0 + ((long long)(c + 1) * (kv1 - kv0)) / n_chunks;
    steps += (b - a + BLOCK_N - 1) / BLOCK_N;
    aligned = aligned && (b - a) % BLOCK_N == 0;
  }
  const bool qtm = steps >= 24;
  // merge mode with head dims up to 80 stages the accumulated rows in shared memory
#define ST_SPATIAL(DD, MM, QQ)                                                                                   \
  (ring ? (aligned ? launch_spatial<DD, false, 2, QQ>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s, o_acc,   \
                                                     lse_acc, n_chunks, ring)                                   \
                   : launch_spatial<DD, false, 1, QQ>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s, o_acc,   \
                                                     lse_acc, n_chunks, ring))                                  \
        : launch_spatial<DD, MM, 0, QQ>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s, o_acc, lse_acc,      \
                                        n_chunks, ring))
  const bool staged = o_acc != nullptr;
  switch (g.D) {
    case 32: return staged ? ST_SPATIAL(32, true, false) : ST_SPATIAL(32, false, false);
    case 64: return staged ? ST_SPATIAL(64, true, false) : ST_SPATIAL(64, false, false);
    case 72:
      if (qtm) return staged ? ST_SPATIAL(72, true, true) : ST_SPATIAL(72, false, true);
      return staged ? ST_SPATIAL(72, true, false) : ST_SPATIAL(72, false, false);
    case 80:
      if (qtm) return staged ? ST_SPATIAL(80, true, true) : ST_SPATIAL(80, false, true);
      return staged ? ST_SPATIAL(80, true, false) : ST_SPATIAL(80, false, false);
    case 96: return ST_SPATIAL(96, false, false);
    case 128: return ST_SPATIAL(128, false, false);
  }
#undef ST_SPATIAL
  return ST_ERR_UNSUPPORTED;
}

}  // namespace st

ST_API st_status st_selftest_ex2(const float *x, float *y_poly, float *y_mufu, int n, st_stream_t stream) {
  if (n < 0) return ST_ERR_SHAPE;
  if (n == 0) return ST_OK;
  if (!x || !y_poly || !y_mufu) return ST_ERR_NULL;
  if (!st::is_aligned(x, 4) || !st::is_aligned(y_poly, 4) || !st::is_aligned(y_mufu, 4)) return ST_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ex2_probe<<<(n + 255) / 256, 256, 0, s>>>(x, y_poly, y_mufu, n);
  return st::launch_status();
}

ST_API st_status st_selftest_wait_timeout(st_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wait_timeout_probe<<<1, 32, 0, s>>>(20000000ull /* 20 ms */, 0u);
  return st::launch_status();
}
