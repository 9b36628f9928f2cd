// ulysses_relayout: the all-to-all of sequence parallelism as an in-HBM
// permutation on a virtual partition of P shards.
//
// Layouts (ScaleFusion review, "三、技术架构" distributed execution flow and
// "四、核心创新" pseudo-code; CoCoDiff article, Ulysses section):
//   x, shard p: [B, N_T, N_S, T/N_T, S/(N_S*P), C]   (spatially sharded)
//   y, shard q: [B, N_T, N_S, T/(N_T*P), S/N_S, C]   (temporally sharded)
//   seq,  shard p: [B, N/P, H, D]                   (sequence sharded)
//   head, shard q: [B, H/P, N, D]                   (head sharded)
//
// Design.  The permutation moves "segments": runs of elements that are
// contiguous in BOTH the source and the destination.  For the spatial/temporal
// exchange a segment is the S/(N_S*P) tokens (x C channels) that one x shard
// holds of one frame of one (i, j) block -- tens to hundreds of KB, so the
// kernel is a strided block copy.  For the sequence/head exchange a segment is
// the D channels of one (token, head).  A group of lanes maps one segment with
// a few integer divisions and then streams it with the widest aligned vector
// (16 bytes when possible), several vectors in flight per lane, in destination
// order.  The optional RMSNorm is a second kernel: the bulk copy engine
// stages 32 heads per warp in shared memory, one lane normalises each head.
#include "common.cuh"

namespace {

struct Map {
  int mode;
  int P, B;
  int n_t, n_s, i0, n_i, j0, n_j;
  int q0, n_q;             // temporally sharded side: shards q0 <= q < q0 + n_q
  int Tn, Tq, Sp, Ss;      // T/N_T, T/(N_T*P), S/(N_S*P), S/N_S
  int N, H, Np, Hp;        // sequence/head exchange
  long long row_bytes;     // bytes per row (C or D elements)
  long long seg_bytes;     // bytes per segment
  long long n_segs;
};

// Byte offsets of segment g in the source and the destination; with pos0,
// the sequence position of the segment's first destination row (S2T: its
// token index s in the frame; SEQ2HEAD: its n).
__device__ __forceinline__ void map_segment(const Map &m, long long g, long long &src,
                                            long long &dst, int *pos0 = nullptr) {
  long long src_row, dst_row;
  if (m.mode == ST_S2T) {
    // segments enumerate destination rows (q, b, i, j, t2, p); p fastest
    int p = int(g % m.P); g /= m.P;
    int t2 = int(g % m.Tq); g /= m.Tq;
    int j = m.j0 + int(g % m.n_j); g /= m.n_j;
    int i = m.i0 + int(g % m.n_i); g /= m.n_i;
    int b = int(g % m.B);
    int q = m.q0 + int(g / m.B);
    long long blk_y = (((long long)q * m.B + b) * m.n_t + i) * m.n_s + j;
    long long blk_x = (((long long)p * m.B + b) * m.n_t + i) * m.n_s + j;
    dst_row = (blk_y * m.Tq + t2) * m.Ss + (long long)p * m.Sp;
    src_row = (blk_x * m.Tn + (long long)q * m.Tq + t2) * m.Sp;
    if (pos0) *pos0 = j * m.Ss + p * m.Sp;
  } else if (m.mode == ST_T2S) {
    // segments enumerate destination rows (p, b, i, j, t1) whose frame comes
    // from the selected y shards: t1 in [q0 * Tq, (q0 + n_q) * Tq)
    const int nt1 = m.n_q * m.Tq;
    int t1 = m.q0 * m.Tq + int(g % nt1); g /= nt1;
    int j = m.j0 + int(g % m.n_j); g /= m.n_j;
    int i = m.i0 + int(g % m.n_i); g /= m.n_i;
    int b = int(g % m.B);
    int p = int(g / m.B);
    int q = t1 / m.Tq, t2 = t1 - q * m.Tq;
    long long blk_y = (((long long)q * m.B + b) * m.n_t + i) * m.n_s + j;
    long long blk_x = (((long long)p * m.B + b) * m.n_t + i) * m.n_s + j;
    dst_row = (blk_x * m.Tn + t1) * m.Sp;
    src_row = (blk_y * m.Tq + t2) * m.Ss + (long long)p * m.Sp;
  } else if (m.mode == ST_SEQ2HEAD) {
    // destination rows (q, b, h1, n); n fastest
    dst_row = g;
    int n = int(g % m.N); g /= m.N;
    if (pos0) *pos0 = n;
    int h1 = int(g % m.Hp); g /= m.Hp;
    int b = int(g % m.B);
    int q = int(g / m.B);
    int p = n / m.Np, n1 = n - p * m.Np;
    src_row = (((long long)p * m.B + b) * m.Np + n1) * m.H + (long long)q * m.Hp + h1;
  } else {
    // ST_HEAD2SEQ: destination rows (p, b, n1, h); h fastest
    dst_row = g;
    int h = int(g % m.H); g /= m.H;
    int n1 = int(g % m.Np); g /= m.Np;
    int b = int(g % m.B);
    int p = int(g / m.B);
    int q = h / m.Hp, h1 = h - q * m.Hp;
    src_row = (((long long)q * m.B + b) * m.Hp + h1) * m.N + (long long)p * m.Np + n1;
  }
  src = src_row * m.row_bytes;
  dst = dst_row * m.row_bytes;
}

template <int VEC> struct VecT;
template <> struct VecT<16> { using t = uint4; };
template <> struct VecT<8> { using t = uint2; };
template <> struct VecT<4> { using t = uint32_t; };
template <> struct VecT<2> { using t = uint16_t; };
template <> struct VecT<1> { using t = uint8_t; };

// Work item = (segment, chunk of G*U consecutive vectors).  A group of G
// lanes handles IU items per iteration, issuing all IU*U loads before the
// stores so that many bytes are in flight per lane.
template <int VEC, int U, int IU>
__global__ void __launch_bounds__(256) relayout_copy(Map m, int G, int log2G,
                                                     const char *__restrict__ in,
                                                     char *__restrict__ out) {
  using V = typename VecT<VEC>::t;
  st::pdl_trigger();
  st::pdl_wait();
  in = st::after_wait(in);
  const long long seg_vecs = m.seg_bytes / VEC;
  const long long chunk = (long long)G * U;
  const long long n_chunks = (seg_vecs + chunk - 1) / chunk;
  const long long n_items = m.n_segs * n_chunks;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = int(tid & (G - 1));
  const long long group = tid >> log2G;
  const long long n_groups = ((long long)gridDim.x * blockDim.x) >> log2G;
  for (long long it0 = group * IU; it0 < n_items; it0 += n_groups * IU) {
    V buf[IU][U];
    long long dst_off[IU];
    long long k0[IU];
#pragma unroll
    for (int iu = 0; iu < IU; ++iu) {
      const long long item = it0 + iu;
      dst_off[iu] = -1;
      if (item < n_items) {
        const long long seg = item / n_chunks;
        const long long ch = item - seg * n_chunks;
        long long s, d;
        map_segment(m, seg, s, d);
        dst_off[iu] = d;
        k0[iu] = ch * chunk + lane;
        const V *src = reinterpret_cast<const V *>(in + s);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const long long k = k0[iu] + (long long)u * G;
          if (k < seg_vecs) buf[iu][u] = __ldg(src + k);
        }
      }
    }
#pragma unroll
    for (int iu = 0; iu < IU; ++iu) {
      if (dst_off[iu] < 0) continue;
      V *dst = reinterpret_cast<V *>(out + dst_off[iu]);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const long long k = k0[iu] + (long long)u * G;
        if (k < seg_vecs) dst[k] = buf[iu][u];
      }
    }
  }
}

// ---------------------------------------------------------------- RMSNorm flavour
//   y_d = x_d / sqrt(mean_d x_d^2 + eps) * gamma_d   (fp32 math)
// A warp task is 32 consecutive heads in destination order.  The bulk copy
// engine brings them into a per-warp shared buffer (one copy when the heads
// are contiguous in the source, as inside a spatial/temporal segment;
// otherwise one copy per head, issued by the heads' lanes), each lane
// normalises one head in place, and one bulk copy writes the 32 heads back.
// Every warp double-buffers: the next task's load is in flight while the
// current one is normalised.  Waits on the copies are bounded in time.
__device__ unsigned int g_relayout_error;

__device__ __forceinline__ uint32_t sh_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(sh_u32(dst)), "l"(src), "r"(bytes), "r"(sh_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(sh_u32(src)),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sh_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_try(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}\n"
               : "=r"(ok)
               : "r"(sh_u32(bar)), "r"(parity)
               : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

constexpr int RMS_WARPS = 4;
constexpr unsigned long long RMS_WAIT_NS = 2000000000ull;

// Five CTAs per SM (20 warps) without the rotation: registers capped for it,
// and the launch asks for the largest shared-memory carveout.
template <typename T, int D, bool ROPE>
__global__ void __launch_bounds__(RMS_WARPS * 32, ROPE ? 1 : 5) relayout_rms(Map m, const char *__restrict__ in,
                                                               char *__restrict__ out,
                                                               const float *__restrict__ gamma, float eps,
                                                               const float2 *__restrict__ rope) {
  constexpr int EPV = 16 / int(sizeof(T));               // elements per 16-byte vector
  constexpr int VPH = D / EPV;                           // vectors per head
  constexpr int HB = D * int(sizeof(T));                 // bytes per head
  constexpr int BUF = 32 * HB;                           // bytes per warp buffer
  constexpr int ROT = VPH % 4 == 0 ? 1 : 0;              // vector rotation per lane: no bank conflicts
  extern __shared__ __align__(128) uint8_t rms_smem[];
  __shared__ uint64_t full[RMS_WARPS][2];
  __shared__ float g_s[D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  in = st::after_wait(in);
  gamma = st::after_wait(gamma);
  if constexpr (ROPE) rope = st::after_wait(rope);
  for (int d = threadIdx.x; d < D; d += blockDim.x) g_s[d] = gamma[d];
  if (lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sh_u32(&full[warp][0])) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sh_u32(&full[warp][1])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint8_t *buf0 = rms_smem + warp * 2 * BUF;
  const bool one_src = (m.mode == ST_S2T || m.mode == ST_T2S);   // heads of a task contiguous in the source
  const long long hps = m.seg_bytes / HB;                         // heads per segment
  const long long tps = one_src ? (hps + 31) / 32 : 1;            // tasks per segment (unused otherwise)
  const int hpr = int(m.row_bytes / HB);                          // heads per row
  const long long n_tasks = one_src ? m.n_segs * tps : (m.n_segs + 31) / 32;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;

  // task -> (destination byte offset, number of heads, sequence position of
  // this lane's head when rotating); issues its load into buffer b
  auto issue = [&](long long task, int b, long long &dst, int &nh, int &pos) {
    uint8_t *bufp = buf0 + b * BUF;
    if (one_src) {
      const long long seg = task / tps;
      const long long c = task - seg * tps;
      nh = int(min(32LL, hps - c * 32));
      long long so, dof;
      int p0 = 0;
      map_segment(m, seg, so, dof, ROPE ? &p0 : nullptr);
      dst = dof + c * 32 * HB;
      // S2T: the segment holds Sp whole destination rows of hpr heads each
      if constexpr (ROPE) pos = p0 + int(c * 32 + lane) / hpr;
      if (lane == 0) {
        expect_tx(&full[warp][b], nh * HB);
        bulk_g2s(bufp, in + so + c * 32 * HB, nh * HB, &full[warp][b]);
      }
    } else {
      const long long g0 = task * 32;
      nh = int(min(32LL, m.n_segs - g0));
      long long so, dof;
      int p0 = 0;
      map_segment(m, g0 + (lane < nh ? lane : 0), so, dof, ROPE ? &p0 : nullptr);
      pos = p0;                                                   // SEQ2HEAD: this lane's row
      dst = __shfl_sync(0xffffffffu, dof, 0);                     // destination rows are consecutive
      if (lane == 0) expect_tx(&full[warp][b], nh * HB);
      __syncwarp();
      if (lane < nh) bulk_g2s(bufp + lane * HB, in + so, HB, &full[warp][b]);
    }
  };

  bool ok = true;
  long long dst_cur = 0, dst_next = 0;
  int nh_cur = 0, nh_next = 0, pos_cur = 0, pos_next = 0;
  if (gw < n_tasks) issue(gw, 0, dst_cur, nh_cur, pos_cur);
  int i = 0;
  for (long long task = gw; task < n_tasks && ok; task += nw, ++i) {
    const int b = i & 1;
    const long long next = task + nw;
    if (next < n_tasks) {
      // the store of the previous task used the other buffer: it must have read it
      if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      __syncwarp();
      issue(next, b ^ 1, dst_next, nh_next, pos_next);
    }
    {
      const unsigned long long t0 = gtimer();
      while (!bar_try(&full[warp][b], (i >> 1) & 1)) {
        if (gtimer() - t0 > RMS_WAIT_NS) {
          atomicOr(&g_relayout_error, 1u);
          ok = false;
          break;
        }
      }
    }
    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    uint8_t *bufp = buf0 + b * BUF;
    if (lane < nh_cur) {
      uint8_t *h = bufp + lane * HB;
      const int r0 = (lane * ROT) % VPH;
      auto uix = [&](int u0) { return u0 + r0 < VPH ? u0 + r0 : u0 + r0 - VPH; };
      // the rotary angles of this head's token: its index s in the frame (S2T)
      // or in the sequence (SEQ2HEAD), a row of the (cos, sin) table; the first
      // group of pairs is on its way during the sum of squares
      const float2 *rot = ROPE ? rope + (long long)pos_cur * (D / 2) : nullptr;
      st::RotVec<T> cs[st::RG];
      if constexpr (ROPE) {
#pragma unroll
        for (int g = 0; g < st::RG && g < VPH; ++g) cs[g] = st::load_rot<T>(rot + uix(g) * (EPV / 2));
      }
      float ss = 0.f;
#pragma unroll
      for (int u0 = 0; u0 < VPH; ++u0) {
        const int u = uix(u0);
        const uint4 v = *reinterpret_cast<const uint4 *>(h + u * 16);
        if constexpr (sizeof(T) == 2) {
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a = __uint_as_float(w[k] << 16), c = __uint_as_float(w[k] & 0xffff0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(c, c, ss);
          }
        } else {
          ss = fmaf(__uint_as_float(v.x), __uint_as_float(v.x), ss);
          ss = fmaf(__uint_as_float(v.y), __uint_as_float(v.y), ss);
          ss = fmaf(__uint_as_float(v.z), __uint_as_float(v.z), ss);
          ss = fmaf(__uint_as_float(v.w), __uint_as_float(v.w), ss);
        }
      }
      const float inv = rsqrtf(ss * (1.0f / float(D)) + eps);
#pragma unroll
      for (int u0 = 0; u0 < VPH; ++u0) {
        if constexpr (ROPE) {
          if (u0 > 0 && u0 % st::RG == 0) {
#pragma unroll
            for (int g = 0; g < st::RG; ++g)
              if (u0 + g < VPH) cs[g] = st::load_rot<T>(rot + uix(u0 + g) * (EPV / 2));
          }
        }
        const int u = uix(u0);
        const uint4 v = *reinterpret_cast<const uint4 *>(h + u * 16);
        *reinterpret_cast<uint4 *>(h + u * 16) = st::rms_rope_vec<T, ROPE>(v, inv, g_s + u * EPV, cs[u0 % st::RG]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) bulk_s2g(out + dst_cur, bufp, nh_cur * HB);
    dst_cur = dst_next;
    nh_cur = nh_next;
    pos_cur = pos_next;
  }
  if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  if (!ok && lane == 0) {
    // a copy into this warp's buffers may still be in flight: wait for it (bounded) before exiting
    const unsigned long long t0 = gtimer();
    for (int it = i; it < i + 2; ++it)   // uses it and it + 1: buffer it & 1, phase (it >> 1) & 1
      while (!bar_try(&full[warp][it & 1], (it >> 1) & 1) && gtimer() - t0 < RMS_WAIT_NS) {
      }
  }
  __syncwarp();
}

template <typename T, int D>
st_status launch_rms_d(const Map &m, const char *in, char *out, const float *gamma, float eps, int sms,
                       cudaStream_t s, const float2 *rope) {
  constexpr int BUF = 32 * D * int(sizeof(T));
  constexpr int SMEM = RMS_WARPS * 2 * BUF;
  auto kern = rope ? relayout_rms<T, D, true> : relayout_rms<T, D, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return ST_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, RMS_WARPS * 32, SMEM) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const bool one_src = (m.mode == ST_S2T || m.mode == ST_T2S);
  const long long hps = m.seg_bytes / (D * (long long)sizeof(T));
  const long long n_tasks = one_src ? m.n_segs * ((hps + 31) / 32) : (m.n_segs + 31) / 32;
  const long long want = (n_tasks + RMS_WARPS - 1) / RMS_WARPS;
  const long long cap = (long long)sms * per_sm;
  const int grid = int(want < cap ? want : cap);
  return st::launch_pdl(kern, grid, RMS_WARPS * 32, SMEM, s, m, in, out, gamma, eps, rope);
}

template <typename T>
st_status launch_rms(const Map &m, const char *in, char *out, const float *gamma, int D, float eps, int sms,
                     cudaStream_t s, const float2 *rope = nullptr) {
  switch (D) {
    case 32: return launch_rms_d<T, 32>(m, in, out, gamma, eps, sms, s, rope);
    case 64: return launch_rms_d<T, 64>(m, in, out, gamma, eps, sms, s, rope);
    case 72: return launch_rms_d<T, 72>(m, in, out, gamma, eps, sms, s, rope);
    case 80: return launch_rms_d<T, 80>(m, in, out, gamma, eps, sms, s, rope);
    case 96: return launch_rms_d<T, 96>(m, in, out, gamma, eps, sms, s, rope);
    case 128: return launch_rms_d<T, 128>(m, in, out, gamma, eps, sms, s, rope);
    default: return ST_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------- sequence <-> head exchange
// Rows of D elements whose byte length is 8, 16 or 32 vectors of 16 bytes
// (VPR).  The kernel walks the SEQUENCE side [P, B, N/P, H, D] -- where the H
// rows of a token are contiguous -- in chunks of 32 * U vectors per warp, in
// order, so that side is read (SEQ2HEAD) or written (HEAD2SEQ) in long runs;
// the other side is addressed row by row: row (q, b, h1, n) of the head side
// is ((q*B + b)*Hp + h1)*N + n.  A warp holds U vectors per lane in flight
// (all loads before any store).  The VPR lanes holding one row are
// consecutive (VPR divides 32), so the optional per-head RMSNorm reduces the
// row's sum of squares with VPR-lane butterfly shuffles; every lane keeps the
// gains of its own columns in registers.  The index arithmetic per vector is
// two multiply-shift divisions (by H and by Hp; and by N/P and B when B > 1).
struct SeqHead {
  uint32_t N, H, Hp, Np, B;
  st::FastDiv div_h, div_hp, div_np, div_b;
  long long n_vecs;          // B * N * H * VPR
};

template <typename T, int VPR, int U, bool RMS, bool TO_HEAD>
__global__ void __launch_bounds__(256, RMS ? 3 : 4) seqhead_move(SeqHead m, const char *__restrict__ in, char *__restrict__ out,
                                                    const float *__restrict__ gamma, float eps) {
  constexpr int EPV = 16 / int(sizeof(T));
  constexpr int LOG_VPR = VPR == 8 ? 3 : (VPR == 16 ? 4 : 5);
  st::pdl_trigger();
  st::pdl_wait();
  in = st::after_wait(in);
  const int lane = threadIdx.x & 31;
  const int col = lane & (VPR - 1);                  // this lane's 16-byte column of every row it touches
  float g[EPV];
  if constexpr (RMS) {
    gamma = st::after_wait(gamma);
#pragma unroll
    for (int e = 0; e < EPV; ++e) g[e] = gamma[col * EPV + e];
  }
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  const long long chunk = 32LL * U;
  for (long long c0 = warp * chunk; c0 < m.n_vecs; c0 += n_warps * chunk) {
    uint4 v[U];
    long long head_off[U];                           // byte offset of the vector on the head side
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long vi = c0 + u * 32 + lane;       // vector index on the sequence side
      head_off[u] = -1;
      if (vi < m.n_vecs) {
        // sequence-side row ((p*B + b)*Np + n1)*H + h holds token n = p*Np + n1, head h
        const uint32_t row = uint32_t(vi >> LOG_VPR);
        const uint32_t t = st::fdiv(row, m.div_h);
        const uint32_t h = row - t * m.H;
        uint32_t b = 0, n = t;                         // B = 1: t = p*Np + n1 = n
        if (m.B > 1) {
          const uint32_t pb = st::fdiv(t, m.div_np);
          const uint32_t p = st::fdiv(pb, m.div_b);
          b = pb - p * m.B;
          n = p * m.Np + (t - pb * m.Np);
        }
        const uint32_t q = st::fdiv(h, m.div_hp), h1 = h - q * m.Hp;
        const long long hrow = ((long long)(q * m.B + b) * m.Hp + h1) * m.N + n;
        head_off[u] = (hrow * VPR + col) * 16;
        const char *src = TO_HEAD ? in + vi * 16 : in + head_off[u];
        v[u] = __ldg(reinterpret_cast<const uint4 *>(src));
      } else {
        v[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if constexpr (RMS) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        float ss = 0.f;
        if constexpr (sizeof(T) == 2) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a = __uint_as_float(w[k] << 16), c = __uint_as_float(w[k] & 0xffff0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(c, c, ss);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) ss = fmaf(__uint_as_float(w[k]), __uint_as_float(w[k]), ss);
        }
#pragma unroll
        for (int off = VPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = rsqrtf(ss * (1.0f / float(VPR * EPV)) + eps);
        st::RotVec<T> none;
        v[u] = st::rms_rope_vec<T, false>(v[u], inv, g, none);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (head_off[u] < 0) continue;
      const long long vi = c0 + u * 32 + lane;
      char *dst = TO_HEAD ? out + head_off[u] : out + vi * 16;
      *reinterpret_cast<uint4 *>(dst) = v[u];
    }
  }
}

template <typename T, int VPR, bool RMS>
st_status launch_seqhead_v(const SeqHead &m, bool to_head, const char *in, char *out, const float *gamma, float eps,
                           int sms, cudaStream_t s) {
  constexpr int U = 8;
  const long long chunks = (m.n_vecs + 32LL * U - 1) / (32LL * U);
  const long long want = (chunks + 7) / 8;           // 8 warps per CTA
  const long long cap = (long long)sms * 8;
  const int grid = int(want < cap ? want : cap);
  return to_head ? st::launch_pdl(seqhead_move<T, VPR, U, RMS, true>, grid, 256, 0, s, m, in, out, gamma, eps)
                 : st::launch_pdl(seqhead_move<T, VPR, U, RMS, false>, grid, 256, 0, s, m, in, out, gamma, eps);
}

// Returns ST_ERR_UNSUPPORTED when the rows do not fit the kernel (the caller
// then takes the general segment kernels).
st_status launch_seqhead(const Map &mp, int B, int elem_bytes, const char *in, char *out, const float *gamma,
                         float eps, int sms, cudaStream_t s) {
  const long long rb = mp.row_bytes;
  const int vpr = int(rb / 16);
  if (rb % 16 || !(vpr == 8 || vpr == 16 || vpr == 32)) return ST_ERR_UNSUPPORTED;
  if (!st::is_aligned(in, 16) || !st::is_aligned(out, 16)) return ST_ERR_UNSUPPORTED;
  const long long rows = (long long)B * mp.N * mp.H;
  if (rows >= (1LL << 31) || (long long)B * mp.N >= (1LL << 31)) return ST_ERR_UNSUPPORTED;   // 32-bit row maths
  if (gamma && elem_bytes != 2 && elem_bytes != 4) return ST_ERR_UNSUPPORTED;
  SeqHead m;
  m.N = uint32_t(mp.N); m.H = uint32_t(mp.H); m.Hp = uint32_t(mp.Hp); m.Np = uint32_t(mp.Np); m.B = uint32_t(B);
  m.div_h = st::make_fastdiv(m.H);
  m.div_hp = st::make_fastdiv(m.Hp);
  m.div_np = st::make_fastdiv(m.Np);
  m.div_b = st::make_fastdiv(m.B);
  m.n_vecs = rows * vpr;
  const bool to_head = mp.mode == ST_SEQ2HEAD;
#define ST_SH(TT, V, R) launch_seqhead_v<TT, V, R>(m, to_head, in, out, gamma, eps, sms, s)
  if (!gamma) {
    switch (vpr) {
      case 8: return ST_SH(uint16_t, 8, false);
      case 16: return ST_SH(uint16_t, 16, false);
      default: return ST_SH(uint16_t, 32, false);
    }
  }
  if (elem_bytes == 2) {
    switch (vpr) {
      case 8: return ST_SH(uint16_t, 8, true);
      case 16: return ST_SH(uint16_t, 16, true);
      default: return ST_SH(uint16_t, 32, true);
    }
  }
  switch (vpr) {
    case 8: return ST_SH(float, 8, true);
    case 16: return ST_SH(float, 16, true);
    default: return ST_SH(float, 32, true);
  }
#undef ST_SH
}

template <int VEC>
st_status launch_copy(const Map &m, const char *in, char *out, int grid, cudaStream_t s) {
  const long long seg_vecs = m.seg_bytes / VEC;
  if (seg_vecs >= 256) return st::launch_pdl(relayout_copy<VEC, 8, 1>, grid, 256, 0, s, m, 32, 5, in, out);
  int G = 1, lg = 0;
  while (G < seg_vecs && G < 32) { G <<= 1; ++lg; }
  if (seg_vecs <= G) return st::launch_pdl(relayout_copy<VEC, 1, 4>, grid, 256, 0, s, m, G, lg, in, out);
  return st::launch_pdl(relayout_copy<VEC, 8, 1>, grid, 256, 0, s, m, G, lg, in, out);
}

}  // namespace

namespace st {
unsigned int read_and_clear_relayout_error(cudaStream_t stream, cudaError_t *err) {
  unsigned int word = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&word, g_relayout_error, sizeof(word), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_relayout_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (err) *err = e;
  return word;
}
}  // namespace st

namespace {
st_status relayout_impl(st_relayout_mode mode, const void *in, void *out, int elem_bytes, int P, int B, int T_or_N,
                        int S_or_H, int C_or_D, int n_t, int n_s, int i0, int i1, int j0, int j1, int q0, int q1,
                        const float *rms_gamma, int rms_head_dim, float rms_eps, const float *rope_table,
                        int rope_positions, st_stream_t stream) {
  if (!in || !out) return ST_ERR_NULL;
  if (!(elem_bytes == 1 || elem_bytes == 2 || elem_bytes == 4 || elem_bytes == 8)) return ST_ERR_DTYPE;
  if (P <= 0 || B <= 0 || T_or_N <= 0 || S_or_H <= 0 || C_or_D <= 0 || n_t <= 0 || n_s <= 0)
    return ST_ERR_SHAPE;
  Map m = {};
  m.mode = mode;
  m.P = P;
  m.B = B;
  long long total_elems = (long long)B * T_or_N * S_or_H * C_or_D;
  if (mode == ST_S2T || mode == ST_T2S) {
    const int T = T_or_N, S = S_or_H, C = C_or_D;
    if (T % (n_t * P) || S % (n_s * P)) return ST_ERR_DIVISIBILITY;
    if (i0 < 0 || i1 > n_t || i0 >= i1 || j0 < 0 || j1 > n_s || j0 >= j1) return ST_ERR_SHAPE;
    if (q0 < 0 || q1 > P || q0 >= q1) return ST_ERR_SHAPE;
    m.n_t = n_t; m.n_s = n_s; m.i0 = i0; m.n_i = i1 - i0; m.j0 = j0; m.n_j = j1 - j0;
    m.q0 = q0; m.n_q = q1 - q0;
    m.Tn = T / n_t; m.Tq = T / (n_t * P); m.Sp = S / (n_s * P); m.Ss = S / n_s;
    m.row_bytes = (long long)C * elem_bytes;
    m.seg_bytes = m.Sp * m.row_bytes;
    m.n_segs = (long long)m.n_q * B * m.n_i * m.n_j * m.Tq * P;
    if (rms_gamma && (rms_head_dim <= 0 || C % rms_head_dim)) return ST_ERR_SHAPE;
  } else if (mode == ST_SEQ2HEAD || mode == ST_HEAD2SEQ) {
    const int N = T_or_N, H = S_or_H, D = C_or_D;
    if (n_t != 1 || n_s != 1 || i0 != 0 || i1 != 1 || j0 != 0 || j1 != 1) return ST_ERR_SHAPE;
    if (q0 != 0 || q1 != P) return ST_ERR_SHAPE;
    if (N % P || H % P) return ST_ERR_DIVISIBILITY;
    m.N = N; m.H = H; m.Np = N / P; m.Hp = H / P;
    m.row_bytes = (long long)D * elem_bytes;
    m.seg_bytes = m.row_bytes;
    m.n_segs = (long long)B * N * H;
    if (rms_gamma && rms_head_dim != D) return ST_ERR_SHAPE;
  } else {
    return ST_ERR_UNSUPPORTED;
  }
  if (total_elems == 0) return ST_OK;
  const char *src = static_cast<const char *>(in);
  char *dst = static_cast<char *>(out);
  const long long total_bytes = total_elems * elem_bytes;
  if (src < dst + total_bytes && dst < src + total_bytes) return ST_ERR_SHAPE;  // overlap
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = st::num_sms();
  if (rms_gamma) {
    if (elem_bytes != 2 && elem_bytes != 4) return ST_ERR_DTYPE;
    if ((rms_head_dim * elem_bytes) % 16 || !st::is_aligned(in, 16) || !st::is_aligned(out, 16) ||
        m.row_bytes % 16)
      return ST_ERR_ALIGN;
    const float2 *rope = nullptr;
    if (rope_table) {
      // rotary angles of the attended sequence: tokens of a frame (S2T) or of the sequence (SEQ2HEAD)
      if (mode != ST_S2T && mode != ST_SEQ2HEAD) return ST_ERR_UNSUPPORTED;
      if (rms_head_dim % 2 || rope_positions < (mode == ST_S2T ? S_or_H : T_or_N)) return ST_ERR_SHAPE;
      if (!st::is_aligned(rope_table, 16)) return ST_ERR_ALIGN;
      rope = reinterpret_cast<const float2 *>(rope_table);
    }
    if (!rope && (mode == ST_SEQ2HEAD || mode == ST_HEAD2SEQ)) {
      const st_status r = launch_seqhead(m, B, elem_bytes, src, dst, rms_gamma, rms_eps, sms, s);
      if (r != ST_ERR_UNSUPPORTED) return r;
    }
    return elem_bytes == 2 ? launch_rms<uint16_t>(m, src, dst, rms_gamma, rms_head_dim, rms_eps, sms, s, rope)
                           : launch_rms<float>(m, src, dst, rms_gamma, rms_head_dim, rms_eps, sms, s, rope);
  }
  if (rope_table) return ST_ERR_NULL;               // the rotation rides on the RMSNorm pass
  if (mode == ST_SEQ2HEAD || mode == ST_HEAD2SEQ) {
    const st_status r = launch_seqhead(m, B, elem_bytes, src, dst, nullptr, 0.f, sms, s);
    if (r != ST_ERR_UNSUPPORTED) return r;
  }
  // widest vector that divides the row pitch and both base addresses
  int vec = 16;
  while (vec > elem_bytes && (m.row_bytes % vec || !st::is_aligned(in, vec) || !st::is_aligned(out, vec)))
    vec >>= 1;
  if (m.row_bytes % vec) return ST_ERR_ALIGN;
  const int grid = sms * 8;
  switch (vec) {
    case 16: return launch_copy<16>(m, src, dst, grid, s);
    case 8: return launch_copy<8>(m, src, dst, grid, s);
    case 4: return launch_copy<4>(m, src, dst, grid, s);
    case 2: return launch_copy<2>(m, src, dst, grid, s);
    default: return launch_copy<1>(m, src, dst, grid, s);
  }
}

// rotation table: (cos, sin) of pos * theta^(-2i/D), computed in double precision
__global__ void rope_table_kernel(long long n, int half, double theta, float2 *out) {
  const long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const long long pos = k / half;
  const int i = int(k - pos * half);
  const double a = double(pos) * pow(theta, -2.0 * double(i) / double(2 * half));
  out[k] = make_float2(float(cos(a)), float(sin(a)));
}
}  // namespace

ST_API st_status ulysses_relayout_range(st_relayout_mode mode, const void *in, void *out, int elem_bytes,
                                        int P, int B, int T_or_N, int S_or_H, int C_or_D, int n_t, int n_s,
                                        int i0, int i1, int j0, int j1, int q0, int q1,
                                        const float *rms_gamma, int rms_head_dim, float rms_eps,
                                        st_stream_t stream) {
  return relayout_impl(mode, in, out, elem_bytes, P, B, T_or_N, S_or_H, C_or_D, n_t, n_s, i0, i1, j0, j1, q0, q1,
                       rms_gamma, rms_head_dim, rms_eps, nullptr, 0, stream);
}

ST_API st_status ulysses_relayout(st_relayout_mode mode, const void *in, void *out, int elem_bytes,
                                  int P, int B, int T_or_N, int S_or_H, int C_or_D, int n_t,
                                  int n_s, int i0, int i1, int j0, int j1, const float *rms_gamma,
                                  int rms_head_dim, float rms_eps, st_stream_t stream) {
  return relayout_impl(mode, in, out, elem_bytes, P, B, T_or_N, S_or_H, C_or_D, n_t, n_s, i0, i1, j0, j1, 0, P,
                       rms_gamma, rms_head_dim, rms_eps, nullptr, 0, stream);
}

ST_API st_status ulysses_relayout_rope(st_relayout_mode mode, const void *in, void *out, int elem_bytes, int P, int B,
                                       int T_or_N, int S_or_H, int C_or_D, int n_t, int n_s, const float *rms_gamma,
                                       int rms_head_dim, float rms_eps, const float *rope_table, int rope_positions,
                                       st_stream_t stream) {
  if (!rms_gamma || !rope_table) return ST_ERR_NULL;
  const int i1 = (mode == ST_S2T || mode == ST_T2S) ? n_t : 1, j1 = (mode == ST_S2T || mode == ST_T2S) ? n_s : 1;
  return relayout_impl(mode, in, out, elem_bytes, P, B, T_or_N, S_or_H, C_or_D, n_t, n_s, 0, i1, 0, j1, 0, P,
                       rms_gamma, rms_head_dim, rms_eps, rope_table, rope_positions, stream);
}

ST_API st_status st_rope_table(int n_pos, int head_dim, float theta, float *table, st_stream_t stream) {
  if (!table) return ST_ERR_NULL;
  if (n_pos <= 0 || head_dim <= 0 || head_dim % 2 || !(theta > 0.f)) return ST_ERR_SHAPE;
  if (!st::is_aligned(table, 8)) return ST_ERR_ALIGN;
  const long long n = (long long)n_pos * (head_dim / 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rope_table_kernel<<<int((n + 255) / 256), 256, 0, s>>>(n, head_dim / 2, double(theta),
                                                         reinterpret_cast<float2 *>(table));
  return st::launch_status();
}
