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
// order.  The optional RMSNorm is a second kernel with one thread per head
// segment (its sum of squares stays in registers).
#include "common.cuh"

namespace {

struct Map {
  int mode;
  int P, B;
  int n_t, n_s, i0, n_i, j0, n_j;
  int Tn, Tq, Sp, Ss;      // T/N_T, T/(N_T*P), S/(N_S*P), S/N_S
  int N, H, Np, Hp;        // sequence/head exchange
  long long row_bytes;     // bytes per row (C or D elements)
  long long seg_bytes;     // bytes per segment
  long long n_segs;
};

// Byte offsets of segment g in the source and the destination.
__device__ __forceinline__ void map_segment(const Map &m, long long g, long long &src,
                                            long long &dst) {
  long long src_row, dst_row;
  if (m.mode == ST_S2T) {
    // segments enumerate destination rows (q, b, i, j, t2, p); p fastest
    int p = int(g % m.P); g /= m.P;
    int t2 = int(g % m.Tq); g /= m.Tq;
    int j = m.j0 + int(g % m.n_j); g /= m.n_j;
    int i = m.i0 + int(g % m.n_i); g /= m.n_i;
    int b = int(g % m.B);
    int q = int(g / m.B);
    long long blk_y = (((long long)q * m.B + b) * m.n_t + i) * m.n_s + j;
    long long blk_x = (((long long)p * m.B + b) * m.n_t + i) * m.n_s + j;
    dst_row = (blk_y * m.Tq + t2) * m.Ss + (long long)p * m.Sp;
    src_row = (blk_x * m.Tn + (long long)q * m.Tq + t2) * m.Sp;
  } else if (m.mode == ST_T2S) {
    // segments enumerate destination rows (p, b, i, j, t1)
    int t1 = int(g % m.Tn); g /= m.Tn;
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

// RMSNorm flavour: one thread per head segment of D elements.
//   y_d = x_d / sqrt(mean_d x_d^2 + eps) * gamma_d   (fp32 math)
template <typename T, int D>
__global__ void __launch_bounds__(256) relayout_rms(Map m, const char *__restrict__ in,
                                                    char *__restrict__ out,
                                                    const float *__restrict__ gamma,
                                                    float eps) {
  constexpr int VPH = D * int(sizeof(T)) / 16;          // 16-byte vectors per head
  constexpr int EPV = 16 / int(sizeof(T));               // elements per vector
  const long long heads_per_seg = m.seg_bytes / (D * (long long)sizeof(T));
  const long long n_heads = m.n_segs * heads_per_seg;
  __shared__ float g_s[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) g_s[d] = gamma[d];
  __syncthreads();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long hi = (long long)blockIdx.x * blockDim.x + threadIdx.x; hi < n_heads; hi += stride) {
    const long long seg = hi / heads_per_seg;
    const long long r = hi - seg * heads_per_seg;
    long long s, d;
    map_segment(m, seg, s, d);
    const long long off = r * D * (long long)sizeof(T);
    const uint4 *src = reinterpret_cast<const uint4 *>(in + s + off);
    uint4 *dst = reinterpret_cast<uint4 *>(out + d + off);
    uint4 v[VPH];
#pragma unroll
    for (int u = 0; u < VPH; ++u) v[u] = __ldg(src + u);
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < VPH; ++u) {
      const T *e = reinterpret_cast<const T *>(&v[u]);
#pragma unroll
      for (int k = 0; k < EPV; ++k) {
        float x;
        if constexpr (sizeof(T) == 2) x = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(e)[k]);
        else x = reinterpret_cast<const float *>(e)[k];
        ss = fmaf(x, x, ss);
      }
    }
    const float inv = 1.0f / sqrtf(ss / float(D) + eps);
#pragma unroll
    for (int u = 0; u < VPH; ++u) {
      if constexpr (sizeof(T) == 2) {
        uint16_t *e = reinterpret_cast<uint16_t *>(&v[u]);
#pragma unroll
        for (int k = 0; k < EPV; ++k)
          e[k] = st::f32_to_bf16(st::bf16_to_f32(e[k]) * inv * g_s[u * EPV + k]);
      } else {
        float *e = reinterpret_cast<float *>(&v[u]);
#pragma unroll
        for (int k = 0; k < EPV; ++k) e[k] = e[k] * inv * g_s[u * EPV + k];
      }
      dst[u] = v[u];
    }
  }
}

template <typename T>
st_status launch_rms(const Map &m, const char *in, char *out, const float *gamma, int D,
                     float eps, int grid, cudaStream_t s) {
  switch (D) {
    case 32: relayout_rms<T, 32><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    case 64: relayout_rms<T, 64><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    case 72: relayout_rms<T, 72><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    case 80: relayout_rms<T, 80><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    case 96: relayout_rms<T, 96><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    case 128: relayout_rms<T, 128><<<grid, 256, 0, s>>>(m, in, out, gamma, eps); break;
    default: return ST_ERR_UNSUPPORTED;
  }
  return st::launch_status();
}

template <int VEC>
st_status launch_copy(const Map &m, const char *in, char *out, int grid, cudaStream_t s) {
  const long long seg_vecs = m.seg_bytes / VEC;
  if (seg_vecs >= 256) {
    relayout_copy<VEC, 8, 1><<<grid, 256, 0, s>>>(m, 32, 5, in, out);
  } else {
    int G = 1, lg = 0;
    while (G < seg_vecs && G < 32) { G <<= 1; ++lg; }
    if (seg_vecs <= G) relayout_copy<VEC, 1, 4><<<grid, 256, 0, s>>>(m, G, lg, in, out);
    else relayout_copy<VEC, 8, 1><<<grid, 256, 0, s>>>(m, G, lg, in, out);
  }
  return st::launch_status();
}

}  // namespace

ST_API st_status ulysses_relayout(st_relayout_mode mode, const void *in, void *out, int elem_bytes,
                                  int P, int B, int T_or_N, int S_or_H, int C_or_D, int n_t,
                                  int n_s, int i0, int i1, int j0, int j1, const float *rms_gamma,
                                  int rms_head_dim, float rms_eps, st_stream_t stream) {
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
    m.n_t = n_t; m.n_s = n_s; m.i0 = i0; m.n_i = i1 - i0; m.j0 = j0; m.n_j = j1 - j0;
    m.Tn = T / n_t; m.Tq = T / (n_t * P); m.Sp = S / (n_s * P); m.Ss = S / n_s;
    m.row_bytes = (long long)C * elem_bytes;
    m.seg_bytes = m.Sp * m.row_bytes;
    m.n_segs = (long long)P * B * m.n_i * m.n_j * m.Tn;
    if (rms_gamma && (rms_head_dim <= 0 || C % rms_head_dim)) return ST_ERR_SHAPE;
  } else if (mode == ST_SEQ2HEAD || mode == ST_HEAD2SEQ) {
    const int N = T_or_N, H = S_or_H, D = C_or_D;
    if (n_t != 1 || n_s != 1 || i0 != 0 || i1 != 1 || j0 != 0 || j1 != 1) return ST_ERR_SHAPE;
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
    const long long n_heads = m.n_segs * (m.seg_bytes / ((long long)rms_head_dim * elem_bytes));
    const long long want = (n_heads + 255) / 256;
    const int grid = int(want < (long long)sms * 16 ? want : (long long)sms * 16);
    return elem_bytes == 2 ? launch_rms<uint16_t>(m, src, dst, rms_gamma, rms_head_dim, rms_eps, grid, s)
                           : launch_rms<float>(m, src, dst, rms_gamma, rms_head_dim, rms_eps, grid, s);
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
