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
// threads of the row hit the same cache lines), computes the R weights once,
// then issues all R 16-byte partial loads before the FMAs.  Output is fp32
// or bf16 (rounded once, to nearest even).
#include <math.h>

#include "common.cuh"

namespace {

constexpr int MAXC = 16;

struct MergeArgs {
  const float4 *o[MAXC];
  const float *lse[MAXC];
};

template <bool BF16, int R>
__global__ void __launch_bounds__(256) merge_kernel(MergeArgs a, int nc, long long n_rows_h, int S,
                                                    int H, int D4, void *__restrict__ o_out,
                                                    float *__restrict__ lse_out) {
  const int n = R > 0 ? R : nc;
  const long long total = n_rows_h * D4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long f = (long long)blockIdx.x * blockDim.x + threadIdx.x; f < total; f += stride) {
    const long long rh = f / D4;             // (unit, s, h) row index
    const int d4 = int(f - rh * D4);
    const long long row = rh / H;            // unit * S + s
    const int h = int(rh - row * H);
    const long long unit = row / S;
    const int s = int(row - unit * S);
    const long long li = (unit * H + h) * S + s;
    float l[MAXC];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < (R > 0 ? R : MAXC); ++c) {
      if (c < n) {
        l[c] = __ldg(a.lse[c] + li);
        M = fmaxf(M, l[c]);
      }
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float sum = 0.f;
      float4 v[R > 0 ? R : MAXC];
#pragma unroll
      for (int c = 0; c < (R > 0 ? R : MAXC); ++c)
        if (c < n) v[c] = __ldg(a.o[c] + f);
#pragma unroll
      for (int c = 0; c < (R > 0 ? R : MAXC); ++c)
        if (c < n) sum += expf(l[c] - M);
      lse = M + logf(sum);
#pragma unroll
      for (int c = 0; c < (R > 0 ? R : MAXC); ++c) {
        if (c < n) {
          const float w = expf(l[c] - lse);
          acc.x = fmaf(w, v[c].x, acc.x);
          acc.y = fmaf(w, v[c].y, acc.y);
          acc.z = fmaf(w, v[c].z, acc.z);
          acc.w = fmaf(w, v[c].w, acc.w);
        }
      }
    }
    if (BF16) {
      uint2 p;
      p.x = st::pack_bf16x2(acc.x, acc.y);
      p.y = st::pack_bf16x2(acc.z, acc.w);
      reinterpret_cast<uint2 *>(o_out)[f] = p;
    } else {
      reinterpret_cast<float4 *>(o_out)[f] = acc;
    }
    if (lse_out && d4 == 0) lse_out[li] = lse;
  }
}

template <bool BF16>
void launch(const MergeArgs &a, int nc, long long rows_h, int S, int H, int D4, void *o, float *lse,
            int grid, cudaStream_t s) {
  switch (nc) {
    case 1: merge_kernel<BF16, 1><<<grid, 256, 0, s>>>(a, nc, rows_h, S, H, D4, o, lse); break;
    case 2: merge_kernel<BF16, 2><<<grid, 256, 0, s>>>(a, nc, rows_h, S, H, D4, o, lse); break;
    case 4: merge_kernel<BF16, 4><<<grid, 256, 0, s>>>(a, nc, rows_h, S, H, D4, o, lse); break;
    case 8: merge_kernel<BF16, 8><<<grid, 256, 0, s>>>(a, nc, rows_h, S, H, D4, o, lse); break;
    default: merge_kernel<BF16, 0><<<grid, 256, 0, s>>>(a, nc, rows_h, S, H, D4, o, lse); break;
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
  const long long total = rows_h * (D / 4);
  const long long want = (total + 255) / 256;
  const long long cap = (long long)st::num_sms() * 16;
  const int grid = int(want < cap ? want : cap);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (out_dtype == ST_BF16) launch<true>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s);
  else launch<false>(a, n_chunks, rows_h, S, H, D / 4, o_out, lse_out, grid, s);
  return st::launch_status();
}
