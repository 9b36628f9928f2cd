// Spatial / full attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, per (b, t, head), O = softmax(Q K^T * scale) V over the S tokens
// of frame t (ScaleFusion review, "三、技术架构": the spatial layer; with T = 1
// it is the image-DiT full attention of the xDiT summary, section 3), or the
// normalised partial over one key range [kv0, kv1) plus its log-sum-exp, the
// per-chunk step of ring / Torus attention (SwiftFusion summary,
// Methodology 2).
//
// Design (one CTA per SM, warp-specialised, 10 warps):
//   * A CTA owns 256 query rows of one (b, t, head) as two 128-row tiles A
//     and B.  Q tiles stay resident in shared memory; K and V tiles of 128
//     keys stream through an NS-deep ring of TMA loads (warp 8).
//   * Warp 9 issues the tensor-core work from one thread: S = Q K^T into
//     TMEM (fp32, 128 columns per tile), and O += P V with P read straight
//     from TMEM (the "TS" form), O accumulating in TMEM.  Issue order
//     S_A(j+1) right after PV_A(j) and S_B(j+1) right after PV_B(j) keeps the
//     tensor pipe busy with one tile while the other tile's softmax runs.
//   * Warps 0-3 (tile A) and 4-7 (tile B) are the softmax warpgroups: one
//     thread per query row (TMEM lane), 128 scores per row loaded with
//     tcgen05.ld, row max, exp2 with the softmax scale folded in, row sum in
//     fp32, P packed to bf16 and written back over the S columns.  The
//     running max is only raised (and O rescaled in TMEM) when it grows by
//     more than 2^8, so the O correction is rare.
//   * The epilogue divides by the row sum, rounds once to bf16 (or keeps fp32
//     partials) and writes each row, plus the natural-log LSE.
//   * Head dims 32..128: the D axis is split into a 64-wide 128B-swizzled
//     chunk and a remainder chunk padded to 16/32/64 (zero-filled by TMA
//     beyond D), each with its own swizzle mode, so D = 72 costs K = 80.
//   * Every wait on an mbarrier is bounded (wall clock).  A wait that runs out
//     records its site in a device error word, raises an abort epoch that
//     makes every other wait of the same launch give up, drains in-flight
//     copies and MMAs, frees TMEM and exits; the host reports ST_ERR_TIMEOUT.
#include <cuda.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "attn_geom.cuh"

namespace {

__device__ unsigned int g_attn_error;        // sites of waits that ran out
__device__ unsigned int g_attn_abort_epoch;  // launch epoch that must abort

constexpr int NUM_THREADS = 320;
constexpr int BLOCK_M = 128;                 // rows per tile
constexpr int BLOCK_N = 128;                 // keys per K/V tile
constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s per wait

template <int D> struct Cfg {
  static constexpr int C0 = D >= 64 ? 64 : 32;
  static constexpr int R1 = D > 64 ? D - 64 : 0;
  static constexpr int C1 = R1 == 0 ? 0 : (R1 <= 16 ? 16 : (R1 <= 32 ? 32 : 64));
  static constexpr int DP = C0 + C1;                   // padded head dim
  static constexpr int SW0 = C0 * 2, SW1 = C1 * 2;     // row bytes = swizzle span
  static constexpr int T0 = BLOCK_M * SW0, T1 = BLOCK_M * SW1;
  static constexpr int TILE = T0 + T1;                 // bytes of one Q/K/V tile
  static constexpr int NS_RAW = (204800 - 2 * TILE) / (2 * TILE);
  static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;   // K/V ring depth
  static constexpr int SMEM = 1024 + 2 * TILE + 2 * NS * TILE + 256;
  static_assert(DP <= 128, "head dim too large");
  static_assert(NS >= 2, "ring too shallow");
};

// ---------------------------------------------------------------- exp2
// 2^x on the special-function unit (one MUFU op, flush-to-zero).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, for x <= 8.  Range reduction x = j + f with j the
// nearest integer (adding 1.5 * 2^23 leaves j in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose coefficients were
// fitted for this kernel by a Remez exchange on relative error over
// [-1/2, 1/2] (max relative error 7.5e-5, far below the bf16 rounding of P);
// 2^j is added into the exponent field.  x is clamped at -125 so the result
// stays a normal number (masked scores give 2^-125, i.e. 0 for all purposes).
constexpr float kP0 = 0.9999280571937561f, kP1 = 0.6932609677314758f;
constexpr float kP2 = 0.2426111251115799f, kP3 = 0.0551716685295105f;
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(kP3, f, kP2), f, kP1), f, kP0);
  return __int_as_float(__float_as_int(p) + ((__float_as_int(t) - 0x4B400000) << 23));
}

// Of every 8 consecutive score pairs, this many take ex2_poly and the rest the
// MUFU, so the two pipes share the exponentials of the softmax.
constexpr int kPolyPairs = 3;

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

// Bounded wait for the phase of the given parity to complete.
__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t epoch, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*reinterpret_cast<volatile unsigned int *>(&g_attn_abort_epoch) == epoch) return false;
      if (globaltimer() - t0 > WAIT_NS) {
        atomicOr(&g_attn_error, 1u << (site & 31));
        atomicExch(&g_attn_abort_epoch, epoch);
        return false;
      }
    }
  }
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
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format): start, LBO, SBO in bytes,
// layout 2 = 128B swizzle, 4 = 64B, 6 = 32B.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                      // descriptor version for sm_100
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
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
  int q_blocks;              // ceil(S / 256)
  int tmode;                 // 1: frames addressed as (t % tblk, b*T/tblk + t/tblk)
  float scale_log2, scale;
  void *o;
  float *lse;
  int o_f32;
  uint32_t epoch;
};

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                   const __grid_constant__ CUtensorMap tk0, const __grid_constant__ CUtensorMap tk1,
                   const __grid_constant__ CUtensorMap tv0, const __grid_constant__ CUtensorMap tv1,
                   const Params p) {
  using K = Cfg<D>;
  constexpr int NS = K::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                          // 2 tiles
  uint8_t *sK = sQ + 2 * K::TILE;              // NS tiles
  uint8_t *sV = sK + NS * K::TILE;             // NS tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sV + NS * K::TILE);
  uint64_t *q_full = bars;                     // 1
  uint64_t *k_full = bars + 1;                 // NS
  uint64_t *k_empty = k_full + NS;             // NS
  uint64_t *v_full = k_empty + NS;             // NS
  uint64_t *v_empty = v_full + NS;             // NS
  uint64_t *s_full = v_empty + NS;             // 2
  uint64_t *p_full = s_full + 2;               // 2
  uint64_t *o_full = p_full + 2;               // 2
  uint64_t *mma_done = o_full + 2;             // 1
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const st::Geom &g = p.g;

  // ---- work item: (q block, head, frame), q block fastest so that the CTAs
  //      that run together share K/V tiles in L2
  int x = blockIdx.x;
  const int qb = x % p.q_blocks;
  x /= p.q_blocks;
  const int h = x % g.H;
  x /= g.H;
  const int t = p.lo + x % p.n_frames;
  const int b = x / p.n_frames;
  const int q0 = qb * 2 * BLOCK_M;
  const int n_qt = (g.S - q0) > BLOCK_M ? 2 : 1;
  const int n_kv = (p.kv1 - p.kv0 + BLOCK_N - 1) / BLOCK_N;
  int c3, c4;
  if (p.tmode) {
    c3 = t % g.tblk;
    c4 = b * (g.T / g.tblk) + t / g.tblk;
  } else {
    c3 = t;
    c4 = b;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, BLOCK_M);
      mbar_init(o_full + i, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
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

  if (warp == 8) {
    // ================= TMA producer =================
    if (lane == 0 && n_kv > 0) {
      bool ok = true;
      int issued = 0;  // K/V loads issued (each j issues one K and one V)
      mbar_expect_tx(q_full, n_qt * K::TILE);
      for (int X = 0; X < n_qt; ++X) {
        uint8_t *dst = sQ + X * K::TILE;
        tma_load_5d(dst, &tq0, q_full, 0, h, q0 + X * BLOCK_M, c3, c4);
        if (K::C1) tma_load_5d(dst + K::T0, &tq1, q_full, 64, h, q0 + X * BLOCK_M, c3, c4);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % NS;
        const uint32_t ph = (j / NS) & 1;
        const int key = p.kv0 + j * BLOCK_N;
        if (!(ok = mbar_wait(k_empty + st, ph ^ 1, epoch, 0))) break;
        mbar_expect_tx(k_full + st, K::TILE);
        uint8_t *dk = sK + st * K::TILE;
        tma_load_5d(dk, &tk0, k_full + st, 0, h, key, c3, c4);
        if (K::C1) tma_load_5d(dk + K::T0, &tk1, k_full + st, 64, h, key, c3, c4);
        if (!(ok = mbar_wait(v_empty + st, ph ^ 1, epoch, 1))) { issued = 2 * j + 1; break; }
        mbar_expect_tx(v_full + st, K::TILE);
        uint8_t *dv = sV + st * K::TILE;
        tma_load_5d(dv, &tv0, v_full + st, 0, h, key, c3, c4);
        if (K::C1) tma_load_5d(dv + K::T0, &tv1, v_full + st, 64, h, key, c3, c4);
        issued = 2 * (j + 1);
      }
      if (!ok) {
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
        // drain: wait (bounded, ignoring the abort epoch) for the last loads issued
        const unsigned long long t0 = globaltimer();
        for (int i = (issued > 2 * NS ? issued - 2 * NS : 0); i < issued; ++i) {
          const int j = i >> 1;
          uint64_t *bar = (i & 1) ? v_full + (j % NS) : k_full + (j % NS);
          const uint32_t ph = (j / NS) & 1;
          while (!mbar_try_wait(bar, ph) && globaltimer() - t0 < WAIT_NS) {
          }
        }
        while (!mbar_try_wait(q_full, 0) && globaltimer() - t0 < WAIT_NS) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================= MMA issuer =================
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t IDS = idesc_bf16(BLOCK_M, BLOCK_N, 0, 0);
      constexpr uint32_t IDP0 = idesc_bf16(BLOCK_M, K::C0, 0, 1);
      constexpr uint32_t IDP1 = idesc_bf16(BLOCK_M, K::C1 ? K::C1 : 16, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      auto issue_s = [&](int X, int st) {
        const uint32_t d = tmem + X * 128;
        const uint32_t qa = aQ + X * K::TILE, ka = aK + st * K::TILE;
#pragma unroll
        for (int kk = 0; kk < K::C0 / 16; ++kk)
          mma_ss(d, sdesc(qa + kk * 32, 16, 8 * K::SW0, layout_of(K::SW0)),
                 sdesc(ka + kk * 32, 16, 8 * K::SW0, layout_of(K::SW0)), IDS, kk > 0);
        if (K::C1) {
#pragma unroll
          for (int kk = 0; kk < (K::C1 ? K::C1 : 16) / 16; ++kk)
            mma_ss(d, sdesc(qa + K::T0 + kk * 32, 16, 8 * K::SW1, layout_of(K::SW1)),
                   sdesc(ka + K::T0 + kk * 32, 16, 8 * K::SW1, layout_of(K::SW1)), IDS, 1);
        }
      };
      auto issue_pv = [&](int X, int st, bool acc) {
        const uint32_t d = tmem + 256 + X * 128;
        const uint32_t pa = tmem + X * 128;  // P (bf16 pairs) over the S columns
        const uint32_t va = aV + st * K::TILE;
#pragma unroll
        for (int kk = 0; kk < BLOCK_N / 16; ++kk) {
          mma_ts(d, pa + kk * 8, sdesc(va + kk * 16 * K::SW0, K::T0, 8 * K::SW0, layout_of(K::SW0)), IDP0,
                 (acc || kk > 0) ? 1u : 0u);
          if (K::C1)
            mma_ts(d + K::C0, pa + kk * 8,
                   sdesc(va + K::T0 + kk * 16 * K::SW1, K::T1, 8 * K::SW1, layout_of(K::SW1)), IDP1,
                   (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, epoch, 2) && mbar_wait(k_full, 0, epoch, 3);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        tc_commit(s_full + 0);
        if (n_qt == 2) {
          issue_s(1, 0);
          tc_commit(s_full + 1);
        }
        tc_commit(k_empty + 0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % NS;
        const uint32_t ph = (j / NS) & 1;
        const bool more = j + 1 < n_kv;
        const int st1 = (j + 1) % NS;
        const uint32_t ph1 = ((j + 1) / NS) & 1;
        if (!(ok = mbar_wait(v_full + st, ph, epoch, 4))) break;
        if (!(ok = mbar_wait(p_full + 0, j & 1, epoch, 5))) break;
        tc_fence_after();
        issue_pv(0, st, j > 0);
        if (more) {
          if (!(ok = mbar_wait(k_full + st1, ph1, epoch, 6))) break;
          tc_fence_after();
          issue_s(0, st1);
          tc_commit(s_full + 0);
        }
        if (n_qt == 2) {
          if (!(ok = mbar_wait(p_full + 1, j & 1, epoch, 7))) break;
          tc_fence_after();
          issue_pv(1, st, j > 0);
          if (more) {
            issue_s(1, st1);
            tc_commit(s_full + 1);
          }
        }
        if (more) tc_commit(k_empty + st1);
        tc_commit(v_empty + st);
      }
      if (ok) {
        tc_commit(o_full + 0);
        if (n_qt == 2) tc_commit(o_full + 1);
      } else {
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
      }
      // every MMA issued by this thread completes before TMEM is released
      tc_commit(mma_done);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(mma_done, 0) && globaltimer() - t0 < WAIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // ================= softmax warpgroups =================
    const int X = warp >> 2;                   // tile
    const int r = ((warp & 3) << 5) + lane;    // row in tile == TMEM lane
    const int qrow = q0 + X * BLOCK_M + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + X * 128;
    const uint32_t tO = tmem + lane_off + 256 + X * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (X < n_qt && n_kv > 0) {
      for (int j = 0; j < n_kv; ++j) {
        if (!(ok = mbar_wait(s_full + X, j & 1, epoch, 8 + X))) break;
        tc_fence_after();
        uint32_t sr[BLOCK_N];
#pragma unroll
        for (int c = 0; c < BLOCK_N / 16; ++c) TMEM_LD16(tS + c * 16, (sr + c * 16));
        tmem_wait_ld();
        const int nvalid = p.kv1 - (p.kv0 + j * BLOCK_N);
        if (nvalid < BLOCK_N) {
#pragma unroll
          for (int c = 0; c < BLOCK_N; ++c)
            if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
        }
        float mxp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mxp[e] = __uint_as_float(sr[e]);
#pragma unroll
        for (int c = 8; c < BLOCK_N; ++c) mxp[c & 7] = fmaxf(mxp[c & 7], __uint_as_float(sr[c]));
        float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                         fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
        mx *= p.scale_log2;
        if (j == 0) {
          m = mx;
        } else {
          const bool need = mx > m + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            const float corr = need ? exp2f(m - mx) : 1.0f;
            if (need) {
              l *= corr;
              m = mx;
            }
#pragma unroll
            for (int c = 0; c < K::DP / 16; ++c) {
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
        float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c0 = 0; c0 < BLOCK_N; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float x0 = fmaf(__uint_as_float(sr[c0 + c]), p.scale_log2, -m);
            const float x1 = fmaf(__uint_as_float(sr[c0 + c + 1]), p.scale_log2, -m);
            float e0, e1;
            if (((c >> 1) & 7) < kPolyPairs) {
              e0 = ex2_poly(x0);
              e1 = ex2_poly(x1);
            } else {
              e0 = ex2_mufu(x0);
              e1 = ex2_mufu(x1);
            }
            sp[(c >> 1) & 7] += e0 + e1;
            pk[c >> 1] = st::pack_bf16x2(e0, e1);
          }
          TMEM_ST16(tS + (c0 >> 1), pk);
        }
        l += ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + X);
      }
      if (ok) ok = mbar_wait(o_full + X, 0, epoch, 10 + X);
      if (ok) {
        tc_fence_after();
        const float inv = 1.0f / l;
        const bool valid = qrow < g.S;
        const long long off = g.frame(b, t) + g.token(valid ? qrow : 0) + (long long)h * D;
#pragma unroll
        for (int c = 0; c < K::DP / 16; ++c) {
          uint32_t ov[16];
          TMEM_LD16(tO + c * 16, ov);
          tmem_wait_ld();
          if (valid && c * 16 < D) {
            if (p.o_f32) {
              float *dst = static_cast<float *>(p.o) + off + c * 16;
#pragma unroll
              for (int e = 0; e < 16; e += 4)
                if (c * 16 + e < D)
                  *reinterpret_cast<float4 *>(dst + e) =
                      make_float4(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv,
                                  __uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
            } else {
              uint16_t *dst = static_cast<uint16_t *>(p.o) + off + c * 16;
#pragma unroll
              for (int e = 0; e < 16; e += 8)
                if (c * 16 + e < D) {
                  uint4 w;
                  w.x = st::pack_bf16x2(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv);
                  w.y = st::pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
                  w.z = st::pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
                  w.w = st::pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
                  *reinterpret_cast<uint4 *>(dst + e) = w;
                }
            }
          }
        }
        if (valid && p.lse)
          p.lse[(((long long)b * g.T + t) * g.H + h) * g.S + qrow] = (m + log2f(l)) * 0.6931471805599453f;
      } else {
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
      }
    } else if (X < n_qt && n_kv == 0) {
      // empty key range: o = 0, lse = -inf
      if (qrow < g.S) {
        const long long off = g.frame(b, t) + g.token(qrow) + (long long)h * D;
        for (int d = 0; d < D; ++d) {
          if (p.o_f32) static_cast<float *>(p.o)[off + d] = 0.f;
          else static_cast<uint16_t *>(p.o)[off + d] = 0;
        }
        if (p.lse) p.lse[(((long long)b * g.T + t) * g.H + h) * g.S + qrow] = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
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

// 5-D map over (d, h, s, frame-in-block, block) with a box of (box_d, 1, 128, 1, 1).
bool make_map(CUtensorMap *m, const void *ptr, const st::Geom &g, int tmode, int box_d, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5], strides[4];
  dims[0] = (cuuint64_t)g.D;
  dims[1] = (cuuint64_t)g.H;
  dims[2] = (cuuint64_t)g.S;
  strides[0] = (cuuint64_t)g.D * 2;
  strides[1] = (cuuint64_t)g.ss * 2;
  if (tmode) {
    dims[3] = (cuuint64_t)g.tblk;
    dims[4] = (cuuint64_t)g.B * (g.T / g.tblk);
    strides[2] = (cuuint64_t)g.st * 2;
    strides[3] = (cuuint64_t)g.stb * 2;
  } else {
    dims[3] = (cuuint64_t)g.T;
    dims[4] = (cuuint64_t)g.B;
    strides[2] = (cuuint64_t)g.st * 2;
    strides[3] = (cuuint64_t)g.sb * 2;
  }
  cuuint32_t box[5] = {(cuuint32_t)box_d, 1, BLOCK_M, 1, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz(swizzle_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

std::atomic<uint32_t> g_epoch{0};

template <int D>
st_status launch_spatial(const st::Geom &g, int lo, int hi, int kv0, int kv1, float scale, const void *q,
                         const void *k, const void *v, void *o, float *lse, int o_f32, cudaStream_t s) {
  using K = Cfg<D>;
  const int tmode = g.tblk != g.T ? 1 : 0;
  CUtensorMap m[6];
  const int c1 = K::C1 ? K::C1 : 16;
  if (!make_map(&m[0], q, g, tmode, K::C0, K::SW0) || !make_map(&m[1], q, g, tmode, c1, c1 * 2) ||
      !make_map(&m[2], k, g, tmode, K::C0, K::SW0) || !make_map(&m[3], k, g, tmode, c1, c1 * 2) ||
      !make_map(&m[4], v, g, tmode, K::C0, K::SW0) || !make_map(&m[5], v, g, tmode, c1, c1 * 2))
    return ST_ERR_CUDA;
  Params p;
  p.g = g;
  p.lo = lo;
  p.n_frames = hi - lo;
  p.kv0 = kv0;
  p.kv1 = kv1;
  p.q_blocks = (g.S + 2 * BLOCK_M - 1) / (2 * BLOCK_M);
  p.tmode = tmode;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o;
  p.lse = lse;
  p.o_f32 = o_f32;
  p.epoch = g_epoch.fetch_add(1) + 1;
  const long long ctas = (long long)p.q_blocks * g.H * g.B * p.n_frames;
  if (ctas <= 0) return ST_OK;
  if (ctas > 0x7fffffffLL) return ST_ERR_SHAPE;
  auto kern = attn_fwd_sm100<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM) != cudaSuccess)
    return ST_ERR_CUDA;
  kern<<<int(ctas), NUM_THREADS, K::SMEM, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], p);
  return st::launch_status();
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
                             const void *k, const void *v, void *o, float *lse, int o_f32, cudaStream_t s) {
  if (hi <= lo) return ST_OK;
  switch (g.D) {
    case 32: return launch_spatial<32>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
    case 64: return launch_spatial<64>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
    case 72: return launch_spatial<72>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
    case 80: return launch_spatial<80>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
    case 96: return launch_spatial<96>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
    case 128: return launch_spatial<128>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_f32, s);
  }
  return ST_ERR_UNSUPPORTED;
}

}  // namespace st

ST_API st_status st_selftest_wait_timeout(st_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wait_timeout_probe<<<1, 32, 0, s>>>(20000000ull /* 20 ms */, 0u);
  return st::launch_status();
}
