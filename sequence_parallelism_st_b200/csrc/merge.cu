// attn_chunk_merge: log-sum-exp merge of the partial results of attention
// over disjoint KV chunks -- the combination step of ring attention and of
// the chunked all-to-all in SwiftFusion's Torus attention (SwiftFusion
// summary, Methodology 2).
//
//   M = max_c lse_c,  lse = M + ln sum_c exp(lse_c - M),  o = sum_c exp(lse_c - lse) o_c
//
// Design.  HBM-bound: every partial element is read once and every output
// written once.  One thread owns four consecutive channels of one
// (unit, token, head) row: it reads the R chunk LSEs of the row (the other
// threads of the row hit the same cache lines) and the R 16-byte partials,
// all issued before any arithmetic (and for two elements at a time), then
// forms the weights as exp(lse_c - M) / sum_c' exp(lse_c' - M): R
// exponentials and one reciprocal; the log only where the LSE is written.  Output is fp32 or bf16 (rounded once, to
// nearest even).
#include <math.h>

#include "common.cuh"

namespace {

constexpr int MAXC = 16;

struct MergeArgs {
  const float4 *o[MAXC];
  const float *lse[MAXC];
};

// Divisors of the row decode, as multiply-shift pairs (32-bit indexing only).
struct MergeDivs {
  st::FastDiv d4, h, s;
};

// Element f of the output (four channels) -> index of its LSE row.
template <typename I>
__device__ __forceinline__ I lse_index(I f, int D4, int H, int S, const MergeDivs &dv) {
  if constexpr (sizeof(I) == 4) {
    const uint32_t rh = st::fdiv(uint32_t(f), dv.d4);   // (unit, s, h) row index
    const uint32_t row = st::fdiv(rh, dv.h);            // unit * S + s
    const uint32_t h = rh - row * uint32_t(H);
    const uint32_t unit = st::fdiv(row, dv.s);
    const uint32_t s = row - unit * uint32_t(S);
    return I((unit * uint32_t(H) + h) * uint32_t(S) + s);
  } else {
    const I rh = f / D4;
    const I row = rh / H;
    const int h = int(rh - row * H);
    const I unit = row / S;
    const int s = int(row - unit * S);
    return (unit * H + h) * S + s;
  }
}

// I is the index type (32-bit when every index fits).  Each thread handles
// U elements per iteration and issues all their loads (R LSEs and R partial
// vectors each) before any arithmetic, so U * 2R loads are in flight.
template <bool BF16, int R, typename I>
__global__ void __launch_bounds__(256) merge_kernel(MergeArgs a, int nc, I n_rows_h, int S, int H, int D4,
                                                    void *__restrict__ o_out, float *__restrict__ lse_out,
                                                    MergeDivs dv) {
  constexpr int NC = R > 0 ? R : MAXC;
  constexpr int U = R > 0 && R <= 4 ? 2 : 1;
  const int n = R > 0 ? R : nc;
  st::pdl_trigger();
  st::pdl_wait();
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (c < n) {
      a.o[c] = st::after_wait(a.o[c]);
      a.lse[c] = st::after_wait(a.lse[c]);
    }
  const I total = n_rows_h * D4;
  const I stride = (I)gridDim.x * blockDim.x;
  for (I f0 = (I)blockIdx.x * blockDim.x + threadIdx.x; f0 < total; f0 += stride * U) {
    float l[U][NC];
    float4 v[U][NC];
    I li[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I f = f0 + (I)u * stride;
      if (f < total) {
        li[u] = lse_index<I>(f, D4, H, S, dv);
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (c < n) {
            l[u][c] = __ldg(a.lse[c] + li[u]);
            v[u][c] = __ldg(a.o[c] + f);
          }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I f = f0 + (I)u * stride;
      if (f >= total) break;
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) M = fmaxf(M, l[u][c]);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float sum = 0.f;
      if (M != -INFINITY) {
        // w_c = exp(lse_c - lse) = e_c / sum_c' e_c' with e_c = exp(lse_c - M)
        float e[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (c < n) {
            e[c] = exp2f((l[u][c] - M) * 1.4426950408889634f);
            sum += e[c];
          }
        const float inv = 1.0f / sum;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          if (c < n) {
            const float w = e[c] * inv;
            acc.x = fmaf(w, v[u][c].x, acc.x);
            acc.y = fmaf(w, v[u][c].y, acc.y);
            acc.z = fmaf(w, v[u][c].z, acc.z);
            acc.w = fmaf(w, v[u][c].w, acc.w);
          }
        }
      }
      if (BF16) {
        uint2 pk;
        pk.x = st::pack_bf16x2(acc.x, acc.y);
        pk.y = st::pack_bf16x2(acc.z, acc.w);
        reinterpret_cast<uint2 *>(o_out)[f] = pk;
      } else {
        reinterpret_cast<float4 *>(o_out)[f] = acc;
      }
      if (lse_out) {
        const bool first = sizeof(I) == 4 ? uint32_t(f) - st::fdiv(uint32_t(f), dv.d4) * uint32_t(D4) == 0
                                          : f % D4 == 0;
        if (first) lse_out[li[u]] = M != -INFINITY ? M + logf(sum) : -INFINITY;
      }
    }
  }
}

template <bool BF16, typename I>
st_status launch(const MergeArgs &a, int nc, long long rows_h, int S, int H, int D4, void *o, float *lse,
                 int grid, cudaStream_t s) {
  const I rh = (I)rows_h;
  const MergeDivs dv{st::make_fastdiv(uint32_t(D4)), st::make_fastdiv(uint32_t(H)), st::make_fastdiv(uint32_t(S))};
  switch (nc) {
    case 1: return st::launch_pdl(merge_kernel<BF16, 1, I>, grid, 256, 0, s, a, nc, rh, S, H, D4, o, lse, dv);
    case 2: return st::launch_pdl(merge_kernel<BF16, 2, I>, grid, 256, 0, s, a, nc, rh, S, H, D4, o, lse, dv);
    case 4: return st::launch_pdl(merge_kernel<BF16, 4, I>, grid, 256, 0, s, a, nc, rh, S, H, D4, o, lse, dv);
    case 8: return st::launch_pdl(merge_kernel<BF16, 8, I>, grid, 256, 0, s, a, nc, rh, S, H, D4, o, lse, dv);
    default: return st::launch_pdl(merge_kernel<BF16, 0, I>, grid, 256, 0, s, a, nc, rh, S, H, D4, o, lse, dv);
  }
}

}  // namespace

ST_API st_status attn_chunk_merge(int n_chunks, const float *const *o_parts, const float *const *lse_parts,
                                  long long n_units, int S, int H, int D, void *o_out, st_dtype out_dtype,
                                  float *lse_out, st_stream_t stream) {
  if (!o_parts || !lse_parts || !o_out) return ST_ERR_NULL;
  if (n_chunks < 1 || n_chunks > MAXC || n_units <= 0 || S <= 0 || H <= 0 || D <= 0) return ST_ERR_SHAPE;
  if (D % 4) return ST_ERR_ALIGN;
  if (out_dtype != ST_F32 && out_dtype != ST_BF16) return ST_ERR_DTYPE;
  MergeArgs a = {};
  for (int c = 0; c < n_chunks; ++c) {
    if (!o_parts[c] || !lse_parts[c]) return ST_ERR_NULL;
    if (!st::is_aligned(o_parts[c], 16) || !st::is_aligned(lse_parts[c], 4)) return ST_ERR_ALIGN;
    a.o[c] = reinterpret_cast<const float4 *>(o_parts[c]);
    a.lse[c] = lse_parts[c];
  }
  if (!st::is_aligned(o_out, out_dtype == ST_BF16 ? 8 : 16)) return ST_ERR_ALIGN;
  const long long rows_h = n_units * S * (long long)H;
  {
    // the outputs are written while other threads (other CTAs) still read
    // the parts: an output that overlaps any part would corrupt the weights
    // or the partials of rows not yet merged
    const long long ob = rows_h * D * (out_dtype == ST_BF16 ? 2 : 4), pb = rows_h * D * 4, lb = rows_h * 4;
    const char *o0 = static_cast<const char *>(o_out), *l0 = reinterpret_cast<const char *>(lse_out);
    auto hit = [](const char *a, long long na, const char *b, long long nb) { return a < b + nb && b < a + na; };
    for (int c = 0; c < n_chunks; ++c) {
      const char *pc = reinterpret_cast<const char *>(o_parts[c]), *lc = reinterpret_cast<const char *>(lse_parts[c]);
      if (hit(o0, ob, pc, pb) || hit(o0, ob, lc, lb)) return ST_ERR_SHAPE;
      if (lse_out && (hit(l0, lb, pc, pb) || hit(l0, lb, lc, lb))) return ST_ERR_SHAPE;
    }
    if (lse_out && hit(o0, ob, l0, lb)) return ST_ERR_SHAPE;
  }
  const long long total = rows_h * (D / 4);
  const long long want = (total + 255) / 256;
  const long long cap = (long long)st::num_sms() * 16;
  const int grid = int(want < cap ? want : cap);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // 32-bit indexing when every element and LSE index (and the loop's overshoot) fits
  const bool small = total + (long long)grid * 256 * 2 < (1LL << 31);
  if (out_dtype == ST_BF16)
    return small ? launch<true, int>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s)
                 : launch<true, long long>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s);
  return small ? launch<false, int>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s)
               : launch<false, long long>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s);
}
