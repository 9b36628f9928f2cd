// Addressing of the [B, T, S, H, D] attention tensors shared by the attention
// kernels, and host-side validation of st_attn_desc.
#pragma once

#include "common.cuh"

namespace st {

// Element (b, t, s, h, d) lives at
//   b*sb + (t / tblk)*stb + (t % tblk)*st + (s / sblk)*ssb + (s % sblk)*ss + h*D + d.
struct Geom {
  int B, T, S, H, D;
  int tblk, sblk;
  long long sb, st, ss, stb, ssb;

  __host__ __device__ __forceinline__ long long frame(int b, int t) const {
    const int tb = t / tblk;
    return (long long)b * sb + (long long)tb * stb + (long long)(t - tb * tblk) * st;
  }
  __host__ __device__ __forceinline__ long long token(int s) const {
    const int q = s / sblk;
    return (long long)q * ssb + (long long)(s - q * sblk) * ss;
  }
};

// Fills g from d (defaults for zero strides), checks sizes and slices, and
// returns the selected range [lo, hi) of frames (spatial) or tokens
// (temporal).
inline st_status make_geom(const st_attn_desc *d, bool temporal, Geom &g, int &lo, int &hi) {
  if (!d) return ST_ERR_NULL;
  if (d->size != (int)sizeof(st_attn_desc)) return ST_ERR_SHAPE;
  if (d->B <= 0 || d->T <= 0 || d->S <= 0 || d->H <= 0 || d->D <= 0) return ST_ERR_SHAPE;
  if (d->dtype != ST_F32 && d->dtype != ST_BF16) return ST_ERR_DTYPE;
  g.B = d->B; g.T = d->T; g.S = d->S; g.H = d->H; g.D = d->D;
  const long long C = (long long)d->H * d->D;
  if (d->t_block < 0 || d->s_block < 0) return ST_ERR_SHAPE;
  if (d->t_block > 0 && d->T % d->t_block) return ST_ERR_DIVISIBILITY;
  if (d->s_block > 0 && d->S % d->s_block) return ST_ERR_DIVISIBILITY;
  g.tblk = d->t_block > 0 ? d->t_block : d->T;
  g.sblk = d->s_block > 0 ? d->s_block : d->S;
  g.ss = d->stride_s ? d->stride_s : C;
  g.ssb = (d->s_block > 0 && d->stride_sb) ? d->stride_sb : (long long)g.sblk * g.ss;
  g.st = d->stride_t ? d->stride_t : (long long)(d->S / g.sblk) * g.ssb;
  g.stb = (d->t_block > 0 && d->stride_tb) ? d->stride_tb : (long long)g.tblk * g.st;
  g.sb = d->stride_b ? d->stride_b : (long long)(d->T / g.tblk) * g.stb;
  if (g.ss < 0 || g.st < 0 || g.sb < 0 || g.ssb < 0 || g.stb < 0) return ST_ERR_SHAPE;
  const int L = temporal ? d->S : d->T;
  lo = 0;
  hi = L;
  if (d->n_slices > 1 && d->slice >= 0) {
    if (L % d->n_slices) return ST_ERR_DIVISIBILITY;
    if (d->slice >= d->n_slices) return ST_ERR_SHAPE;
    lo = d->slice * (L / d->n_slices);
    hi = lo + L / d->n_slices;
  }
  return ST_OK;
}

// Largest element offset touched by the descriptor (+1): used to bound
// the buffers the caller passed.
inline long long geom_extent(const Geom &g) {
  return g.frame(g.B - 1, g.T - 1) + g.token(g.S - 1) + (long long)g.H * g.D;
}

// Entry points of the three attention implementations.
// o_acc / lse_acc (nullable): merge the result with this accumulated partial.
st_status attn_f32(const Geom &g, bool temporal, int lo, int hi, int kv0, int kv1, float scale,
                   const float *q, const float *k, const float *v, float *o, float *lse,
                   cudaStream_t s, const float *o_acc = nullptr, const float *lse_acc = nullptr);
st_status attn_temporal_bf16(const Geom &g, int lo, int hi, float scale, const void *q,
                             const void *k, const void *v, void *o, float *lse, int o_f32,
                             cudaStream_t s);
// n_chunks / ring: the key range cut into n_chunks KV chunks walked in one
// launch; ring = 1 starts every query block at the chunk holding its first row
// (key range = the whole frame, no accumulator).
st_status attn_spatial_sm100(const Geom &g, int lo, int hi, int kv0, int kv1, float scale,
                             const void *q, const void *k, const void *v, void *o, float *lse,
                             int o_f32, cudaStream_t s, const float *o_acc = nullptr,
                             const float *lse_acc = nullptr, int n_chunks = 1, int ring = 0);

}  // namespace st
