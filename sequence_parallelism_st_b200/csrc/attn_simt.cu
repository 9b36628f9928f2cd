// fp32 attention on the fp32 FMA pipes (spatial and temporal units).
//
// Serves the fp32 workloads, whose 1e-4 relative tolerance rules out tf32
// tensor cores.  One warp owns one query row of one unit: each lane holds
// ceil(D/32) channels of q, the dot product with each key is reduced across
// the warp with a fixed butterfly, and the softmax is the online form
// (running max, rescaled running sum and output) in fp32 with expf.
#include <math.h>

#include "attn_geom.cuh"

namespace {

constexpr int MAXR = 4;  // D <= 128

template <bool TEMPORAL>
__global__ void __launch_bounds__(256) attn_f32_kernel(st::Geom g, int lo, int hi, int kv0, int kv1,
                                                       float scale, const float *__restrict__ q,
                                                       const float *__restrict__ k,
                                                       const float *__restrict__ v,
                                                       float *o, float *lse, const float *o_acc,
                                                       const float *lse_acc) {
  const int L = TEMPORAL ? g.T : g.S;            // query rows per unit
  const int nsel = hi - lo;
  const long long n_units = (long long)g.B * nsel * g.H;
  const long long total = n_units * L;
  const int lane = threadIdx.x & 31;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long w = warp0; w < total; w += n_warps) {
    const int row = int(w % L);
    long long u = w / L;
    const int h = int(u % g.H);
    u /= g.H;
    const int sel = lo + int(u % nsel);
    const int b = int(u / nsel);
    // spatial: unit (b, t=sel, h), rows are tokens; temporal: unit (b, s=sel, h), rows are frames
    long long qoff;
    if (TEMPORAL) qoff = g.frame(b, row) + g.token(sel) + (long long)h * g.D;
    else qoff = g.frame(b, sel) + g.token(row) + (long long)h * g.D;
    float qr[MAXR], acc[MAXR];
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      const int d = lane + 32 * r;
      qr[r] = d < g.D ? q[qoff + d] : 0.f;
      acc[r] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const int j0 = TEMPORAL ? 0 : kv0, j1 = TEMPORAL ? g.T : kv1;
    for (int j = j0; j < j1; ++j) {
      long long koff;
      if (TEMPORAL) koff = g.frame(b, j) + g.token(sel) + (long long)h * g.D;
      else koff = g.frame(b, sel) + g.token(j) + (long long)h * g.D;
      float part = 0.f;
#pragma unroll
      for (int r = 0; r < MAXR; ++r) {
        const int d = lane + 32 * r;
        if (d < g.D) part = fmaf(qr[r], k[koff + d], part);
      }
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) part += __shfl_xor_sync(0xffffffffu, part, x);
      const float sc = part * scale;
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn);
      const float p = expf(sc - mn);
      l = l * corr + p;
#pragma unroll
      for (int r = 0; r < MAXR; ++r) {
        const int d = lane + 32 * r;
        acc[r] = acc[r] * corr + (d < g.D ? p * v[koff + d] : 0.f);
      }
      m = mn;
    }
    const long long li = TEMPORAL ? (((long long)b * g.S + sel) * g.H + h) * g.T + row
                                  : (((long long)b * g.T + sel) * g.H + h) * g.S + row;
    float val = l > 0.f ? m + logf(l) : -INFINITY;
    float fa = 0.f, fc = l > 0.f ? 1.f / l : 0.f;
    if (o_acc) {
      // merge with the accumulated partial: weights exp(lse - M) of the two
      const float la = lse_acc[li];
      const float M = fmaxf(la, val);
      if (M != -INFINITY) {
        const float wa = expf(la - M), wc = expf(val - M), sw = wa + wc;
        fa = wa / sw;
        fc = l > 0.f ? wc / (sw * l) : 0.f;
        val = M + logf(sw);
      }
    }
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      const int d = lane + 32 * r;
      if (d < g.D) o[qoff + d] = acc[r] * fc + (o_acc && fa != 0.f ? fa * o_acc[qoff + d] : 0.f);
    }
    if (lse && lane == 0) lse[li] = val;
  }
}

}  // namespace

namespace st {

st_status attn_f32(const Geom &g, bool temporal, int lo, int hi, int kv0, int kv1, float scale,
                   const float *q, const float *k, const float *v, float *o, float *lse,
                   cudaStream_t s, const float *o_acc, const float *lse_acc) {
  if (g.D > 32 * MAXR) return ST_ERR_UNSUPPORTED;
  const long long rows = (long long)g.B * (hi - lo) * g.H * (temporal ? g.T : g.S);
  if (rows == 0) return ST_OK;
  const long long want = (rows * 32 + 255) / 256;
  const long long cap = (long long)num_sms() * 32;
  const int grid = int(want < cap ? want : cap);
  if (temporal)
    attn_f32_kernel<true><<<grid, 256, 0, s>>>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_acc, lse_acc);
  else
    attn_f32_kernel<false><<<grid, 256, 0, s>>>(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, o_acc, lse_acc);
  return launch_status();
}

}  // namespace st
