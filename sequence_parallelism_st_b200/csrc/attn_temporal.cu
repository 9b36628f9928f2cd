// Temporal attention, bf16 in / fp32 accumulate: per (b, s, head) softmax
// attention over the T frames of token s (ScaleFusion review, "三、技术架构":
// the temporal layer attends over dimension T).
//
// Design.  Temporal sequences are short (T <= 64), so the kernel is bound by
// HBM: each token's T rows of Q, K and V are read once and O written once,
// about 16 flop per byte at T = 32.  That is still above what fp32 FMA can
// sustain at HBM speed, so the two small GEMMs run on tensor cores through
// warp-level mma.sync (m16n8k16, plus m16n8k8 for a head dim that is 8 mod
// 16): a unit is far too small for a 128-row tcgen05 tile.
//   * Work item = (token, group of 4 heads); persistent CTAs of 4 warps walk
//     the items with a two-stage cp.async pipeline (the next item's rows load
//     while the current one computes) when two stages fit in 64 KB.  The
//     group's rows are contiguous in HBM (4*D channels), so every frame row
//     is streamed with 16-byte cp.async into a padded shared-memory tile (row
//     pitch 4D+8 elements keeps ldmatrix conflict-free); rows past T are
//     zeroed once.  A thread owns one (tensor, 16-byte column) and walks the
//     frames, whose offsets come from a per-CTA table in shared memory.
//   * Warp w owns head w of the group: S = Q K^T from ldmatrix fragments,
//     row max / row sum by quad shuffles (the warp-shuffle softmax), P kept
//     in registers and re-packed as the A fragment of O = P V (V fragments
//     by ldmatrix.trans), 1/l applied in fp32, one rounding to bf16.
//   * O is staged in the Q tile and written back with coalesced 16-byte
//     stores.
#include <math.h>

#include "attn_geom.cuh"

namespace {

// G: heads per work item and CTA, one warp each (4, or 8 for sequences of at
// most 16 frames, whose items are small)

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x2(uint32_t a, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t a, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(a));
}

__device__ __forceinline__ void mma16816(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma1688(float *c, uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

template <int D, int TP, int STAGES, int G>
__global__ void __launch_bounds__(32 * G) temporal_bf16(st::Geom g, int lo, int n_sel, int n_hg, int n_items,
                                                     float scale_log2, float scale,
                                                     const uint16_t *__restrict__ q,
                                                     const uint16_t *__restrict__ k,
                                                     const uint16_t *__restrict__ v, void *__restrict__ o,
                                                     float *__restrict__ lse, int o_f32) {
  constexpr int RS = G * D + 8;   // shared row pitch (elements)
  constexpr int CH = G * D / 8;   // 16-byte chunks per row
  constexpr int NT = TP / 8;      // key n-tiles
  constexpr int DT = D / 8;       // output n-tiles
  constexpr int KF = D / 16;      // full k16 steps over D
  constexpr int TILE = TP * RS;   // elements of one Q, K or V tile
  extern __shared__ __align__(16) uint16_t smem[];
  // frame offsets of batch 0 (batch b adds b * sb): T entries, so that four
  // single-stage CTAs still fit in an SM whatever B is
  long long *ftab = reinterpret_cast<long long *>(smem + STAGES * 3 * TILE);
  const int T = g.T;
  st::pdl_trigger();
  for (int i = threadIdx.x; i < T; i += blockDim.x) ftab[i] = g.frame(0, i);
  // rows past T are never loaded: zero them once in every tile
  for (int i = threadIdx.x; i < STAGES * 3 * (TP - T) * RS; i += blockDim.x) {
    const int tile = i / ((TP - T) * RS), r = i - tile * (TP - T) * RS;
    smem[tile * TILE + T * RS + r] = 0;
  }
  __syncthreads();
  st::pdl_wait();   // everything above only touched shared memory

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, cq = lane & 3;

  // one item = (b, token s, group of G heads); its Q, K, V rows go to a stage
  auto issue_loads = [&](int item, int stage) {
    const int hg = item % n_hg;
    const int s = lo + (item / n_hg) % n_sel;
    const int b = item / (n_hg * n_sel);
    const int heads_here = min(G, g.H - hg * G);
    const long long tok = g.token(s) + b * g.sb + (long long)hg * G * D;
    const long long *fb = ftab;
    uint16_t *st_base = smem + stage * 3 * TILE;
    // a thread owns a (tensor, 16-byte column) pair and walks the T frames:
    // one shared-table read, one add and one copy per 16 bytes
    const int cols = heads_here * D / 8;
    for (int pc = threadIdx.x; pc < 3 * CH; pc += blockDim.x) {
      const int x = pc / CH, c = pc - x * CH;
      if (c >= cols) continue;
      const uint16_t *src = (x == 0 ? q : (x == 1 ? k : v)) + tok + c * 8;
      uint16_t *dst = st_base + x * TILE + c * 8;
      for (int t = 0; t < T; ++t) cp_async16(dst + t * RS, src + fb[t], 16);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  int stage = 0;
  if (blockIdx.x < n_items) issue_loads(blockIdx.x, 0);
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int next = item + gridDim.x;
    if (STAGES == 2) {
      if (next < n_items) issue_loads(next, stage ^ 1);
      else asm volatile("cp.async.commit_group;\n" ::: "memory");   // keep the group count uniform
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    __syncthreads();
    const int hg = item % n_hg;
    const int s = lo + (item / n_hg) % n_sel;
    const int b = item / (n_hg * n_sel);
    const int heads_here = min(G, g.H - hg * G);
    const long long tok = g.token(s) + b * g.sb + (long long)hg * G * D;
    uint16_t *sQ = smem + stage * 3 * TILE;
    uint16_t *sK = sQ + TILE;
    uint16_t *sV = sK + TILE;
    if (warp < heads_here) {
      const int hcol = warp * D;
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
      for (int mt = 0; mt * 16 < T; ++mt) {
        float sc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
        // S = Q K^T over D
#pragma unroll
        for (int kk = 0; kk < KF; ++kk) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(aQ + 2 * ((mt * 16 + (lane & 15)) * RS + hcol + kk * 16 + (lane >> 4) * 8), a0, a1, a2, a3);
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(aK + 2 * ((np * 16 + (lane & 7) + ((lane >> 4) << 3)) * RS + hcol + kk * 16 +
                              ((lane >> 3) & 1) * 8),
                    b0, b1, b2, b3);
            mma16816(sc[2 * np], a0, a1, a2, a3, b0, b1);
            mma16816(sc[2 * np + 1], a0, a1, a2, a3, b2, b3);
          }
        }
        if constexpr (D % 16 == 8) {
          uint32_t a0, a1;
          ldsm_x2(aQ + 2 * ((mt * 16 + (lane & 15)) * RS + hcol + D - 8), a0, a1);
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t b0, b1;
            ldsm_x2(aK + 2 * ((np * 16 + (lane & 15)) * RS + hcol + D - 8), b0, b1);
            mma1688(sc[2 * np], a0, a1, b0);
            mma1688(sc[2 * np + 1], a0, a1, b1);
          }
        }
        // softmax over keys (rows gq and gq+8 of this m-tile), keys >= T masked
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const int c0 = n * 8 + 2 * cq;
          if (c0 >= T) { sc[n][0] = -INFINITY; sc[n][2] = -INFINITY; }
          if (c0 + 1 >= T) { sc[n][1] = -INFINITY; sc[n][3] = -INFINITY; }
          mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
          mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float off0 = mx0 * scale_log2, off1 = mx1 * scale_log2;
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          sc[n][0] = exp2f(fmaf(sc[n][0], scale_log2, -off0));
          sc[n][1] = exp2f(fmaf(sc[n][1], scale_log2, -off0));
          sc[n][2] = exp2f(fmaf(sc[n][2], scale_log2, -off1));
          sc[n][3] = exp2f(fmaf(sc[n][3], scale_log2, -off1));
          l0 += sc[n][0] + sc[n][1];
          l1 += sc[n][2] + sc[n][3];
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        // O = P V
        float oc[DT][4];
#pragma unroll
        for (int n = 0; n < DT; ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < TP / 16; ++kk) {
          const uint32_t p0 = st::pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
          const uint32_t p1 = st::pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
          const uint32_t p2 = st::pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          const uint32_t p3 = st::pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
          for (int dp = 0; dp < DT / 2; ++dp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(aV + 2 * ((kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RS + hcol + dp * 16 +
                                (lane >> 4) * 8),
                      b0, b1, b2, b3);
            mma16816(oc[2 * dp], p0, p1, p2, p3, b0, b1);
            mma16816(oc[2 * dp + 1], p0, p1, p2, p3, b2, b3);
          }
          if constexpr (DT % 2 == 1) {
            uint32_t b0, b1;
            ldsm_x2_t(aV + 2 * ((kk * 16 + (lane & 15)) * RS + hcol + (DT - 1) * 8), b0, b1);
            mma16816(oc[DT - 1], p0, p1, p2, p3, b0, b1);
          }
        }
        const float i0 = 1.f / l0, i1 = 1.f / l1;
        const int r0 = mt * 16 + gq, r1 = r0 + 8;
        if (!o_f32) {
          // stage O (bf16) in this warp's columns of the Q tile; rows of this m-tile are consumed
#pragma unroll
          for (int n = 0; n < DT; ++n) {
            *reinterpret_cast<uint32_t *>(sQ + r0 * RS + hcol + n * 8 + 2 * cq) =
                st::pack_bf16x2(oc[n][0] * i0, oc[n][1] * i0);
            *reinterpret_cast<uint32_t *>(sQ + r1 * RS + hcol + n * 8 + 2 * cq) =
                st::pack_bf16x2(oc[n][2] * i1, oc[n][3] * i1);
          }
        } else {
          float *of = static_cast<float *>(o);
          const int h = hg * G + warp;
#pragma unroll
          for (int n = 0; n < DT; ++n) {
            if (r0 < T)
              *reinterpret_cast<float2 *>(of + ftab[r0] + tok + warp * D + n * 8 + 2 * cq) =
                  make_float2(oc[n][0] * i0, oc[n][1] * i0);
            if (r1 < T)
              *reinterpret_cast<float2 *>(of + ftab[r1] + tok + warp * D + n * 8 + 2 * cq) =
                  make_float2(oc[n][2] * i1, oc[n][3] * i1);
          }
          (void)h;
        }
        if (lse && cq == 0) {
          const int h = hg * G + warp;
          const long long li = (((long long)b * g.S + s) * g.H + h) * T;
          if (r0 < T) lse[li + r0] = mx0 * scale + logf(l0);
          if (r1 < T) lse[li + r1] = mx1 * scale + logf(l1);
        }
      }
    }
    __syncthreads();
    if (!o_f32) {
      uint16_t *ob = static_cast<uint16_t *>(o);
      const long long *fb = ftab;
      for (int i = threadIdx.x; i < T * CH; i += blockDim.x) {
        const int t = i / CH;
        const int c = i - t * CH;
        if (c * 8 < heads_here * D)
          *reinterpret_cast<uint4 *>(ob + fb[t] + tok + c * 8) = *reinterpret_cast<const uint4 *>(sQ + t * RS + c * 8);
      }
    }
    __syncthreads();   // this stage is refilled two items later
    if (STAGES == 1) {
      if (next < n_items) issue_loads(next, 0);
    } else {
      stage ^= 1;
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

template <int D, int TP>
st_status launch_t(const st::Geom &g, int lo, int n_sel, float scale, const void *q, const void *k,
                   const void *v, void *o, float *lse, int o_f32, cudaStream_t s) {
  // items of 8 heads when the sequence is short (per item the CTA pays three
  // barriers and one pipeline turn; 8 heads of 16 frames move as many bytes as
  // 4 heads of 32), else 4
  constexpr int G = TP <= 16 && D <= 80 ? 8 : 4;
  const int n_hg = (g.H + G - 1) / G;
  const long long items = (long long)g.B * n_sel * n_hg;
  if (items > 0x7fffffffLL) return ST_ERR_SHAPE;
  constexpr size_t stage_bytes = size_t(3) * TP * (G * D + 8) * sizeof(uint16_t);
  // two stages when they fit in 16 KB per warp (the next item's rows load while this one computes)
  constexpr int STAGES = 2 * stage_bytes <= size_t(G) * 16 * 1024 ? 2 : 1;
  const size_t smem = STAGES * stage_bytes + size_t(g.T) * sizeof(long long);
  auto kern = temporal_bf16<D, TP, STAGES, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return ST_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * G, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long cap = (long long)st::num_sms() * per_sm;
  const int grid = int(items < cap ? items : cap);
  const float log2e = 1.4426950408889634f;
  return st::launch_pdl(kern, grid, 32 * G, smem, s, g, lo, n_sel, n_hg, int(items), scale * log2e, scale,
                        static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k),
                        static_cast<const uint16_t *>(v), o, lse, o_f32);
}

template <int D>
st_status launch_d(const st::Geom &g, int lo, int n_sel, float scale, const void *q, const void *k,
                   const void *v, void *o, float *lse, int o_f32, cudaStream_t s) {
  const int tp = (g.T + 15) / 16 * 16;
  switch (tp) {
    case 16: return launch_t<D, 16>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 32: return launch_t<D, 32>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 48: return launch_t<D, 48>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 64: return launch_t<D, 64>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
  }
  return ST_ERR_UNSUPPORTED;
}

}  // namespace

namespace st {

st_status attn_temporal_bf16(const Geom &g, int lo, int hi, float scale, const void *q, const void *k,
                             const void *v, void *o, float *lse, int o_f32, cudaStream_t s) {
  if (g.T > 64) return ST_ERR_UNSUPPORTED;
  const int n_sel = hi - lo;
  if (n_sel <= 0) return ST_OK;
  switch (g.D) {
    case 32: return launch_d<32>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 64: return launch_d<64>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 72: return launch_d<72>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 80: return launch_d<80>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 96: return launch_d<96>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
    case 128: return launch_d<128>(g, lo, n_sel, scale, q, k, v, o, lse, o_f32, s);
  }
  return ST_ERR_UNSUPPORTED;
}

}  // namespace st
