// Public attention entry points: validation and dispatch to the fp32 FMA
// kernel, the bf16 temporal mma kernel or the bf16 tcgen05 spatial kernel.
#include <math.h>

#include "attn_geom.cuh"

namespace {

bool d_supported(int D) { return D == 32 || D == 64 || D == 72 || D == 80 || D == 96 || D == 128; }

// bf16 tensor paths move rows with 16-byte vectors / TMA: every base pointer
// and every stride must be a multiple of 16 bytes.
bool strides_aligned(const st::Geom &g, int esize) {
  const long long a = 16 / esize;
  return g.ss % a == 0 && g.st % a == 0 && g.sb % a == 0 && g.stb % a == 0 && g.ssb % a == 0;
}

}  // namespace

namespace {

st_status spatial(const st_attn_desc *desc, const void *q, const void *k, const void *v, void *o, float *lse,
                  const float *o_acc, const float *lse_acc, st_stream_t stream, int n_chunks = 1, int ring = 0) {
  if (!desc) return ST_ERR_NULL;
  if (!q || !k || !v || !o) return ST_ERR_NULL;
  st::Geom g;
  int lo, hi;
  st_status s = st::make_geom(desc, false, g, lo, hi);
  if (s != ST_OK) return s;
  int kv0 = desc->kv_begin, kv1 = desc->kv_end;
  if (kv0 == 0 && kv1 == 0) kv1 = g.S;
  if (kv0 < 0 || kv1 > g.S || kv0 > kv1) return ST_ERR_SHAPE;
  if (ring && (desc->kv_begin != 0 || desc->kv_end != 0)) return ST_ERR_SHAPE;
  if (n_chunks < 1 || n_chunks > 64 || n_chunks > g.S) return ST_ERR_SHAPE;
  const float scale = desc->scale > 0.f ? desc->scale : 1.0f / sqrtf((float)g.D);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (desc->dtype == ST_F32) {
    if (!st::is_aligned(q, 4) || !st::is_aligned(k, 4) || !st::is_aligned(v, 4) || !st::is_aligned(o, 4))
      return ST_ERR_ALIGN;
    // the fp32 kernel attends the whole range in key order (the same result
    // as the chunk walk up to rounding order)
    return st::attn_f32(g, false, lo, hi, kv0, kv1, scale, static_cast<const float *>(q),
                        static_cast<const float *>(k), static_cast<const float *>(v), static_cast<float *>(o),
                        lse, st, o_acc, lse_acc);
  }
  if (!d_supported(g.D)) return ST_ERR_UNSUPPORTED;
  // the tensor-core kernel needs uniformly strided tokens inside a frame
  if (g.sblk != g.S && g.ssb != (long long)g.sblk * g.ss) return ST_ERR_UNSUPPORTED;
  if (g.tblk != g.T && g.sb != (long long)(g.T / g.tblk) * g.stb) return ST_ERR_UNSUPPORTED;
  if (!st::is_aligned(q, 16) || !st::is_aligned(k, 16) || !st::is_aligned(v, 16) || !st::is_aligned(o, 16))
    return ST_ERR_ALIGN;
  if (o_acc && !st::is_aligned(o_acc, 16)) return ST_ERR_ALIGN;
  if (!strides_aligned(g, 2)) return ST_ERR_ALIGN;
  if (g.sblk != g.S) {                       // uniform in fact: collapse to one level
    g.sblk = g.S;
    g.ssb = (long long)g.S * g.ss;
  }
  return st::attn_spatial_sm100(g, lo, hi, kv0, kv1, scale, q, k, v, o, lse, desc->o_fp32, st, o_acc, lse_acc,
                                n_chunks, ring);
}

}  // namespace

ST_API st_status st_attn_spatial(const st_attn_desc *desc, const void *q, const void *k, const void *v, void *o,
                                 float *lse, st_stream_t stream) {
  return spatial(desc, q, k, v, o, lse, nullptr, nullptr, stream);
}

ST_API st_status st_attn_ring(const st_attn_desc *desc, const void *q, const void *k, const void *v, void *o,
                              float *lse, int n_chunks, st_stream_t stream) {
  return spatial(desc, q, k, v, o, lse, nullptr, nullptr, stream, n_chunks, 1);
}

ST_API st_status st_attn_spatial_merge(const st_attn_desc *desc, const void *q, const void *k, const void *v,
                                       const float *o_acc, const float *lse_acc, void *o, float *lse,
                                       st_stream_t stream) {
  if (!desc || !o_acc || !lse_acc) return ST_ERR_NULL;
  // in place only for an fp32 result (same element layout as the accumulator)
  const bool out_f32 = desc->dtype == ST_F32 || desc->o_fp32;
  if (!out_f32 && static_cast<const void *>(o_acc) == o) return ST_ERR_SHAPE;
  return spatial(desc, q, k, v, o, lse, o_acc, lse_acc, stream);
}

ST_API st_status st_attn_temporal(const st_attn_desc *desc, const void *q, const void *k, const void *v, void *o,
                                  float *lse, st_stream_t stream) {
  if (!desc) return ST_ERR_NULL;
  if (!q || !k || !v || !o) return ST_ERR_NULL;
  st::Geom g;
  int lo, hi;
  st_status s = st::make_geom(desc, true, g, lo, hi);
  if (s != ST_OK) return s;
  if (desc->kv_begin != 0 || desc->kv_end != 0) return ST_ERR_SHAPE;
  const float scale = desc->scale > 0.f ? desc->scale : 1.0f / sqrtf((float)g.D);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (desc->dtype == ST_F32) {
    if (!st::is_aligned(q, 4) || !st::is_aligned(k, 4) || !st::is_aligned(v, 4) || !st::is_aligned(o, 4))
      return ST_ERR_ALIGN;
    return st::attn_f32(g, true, lo, hi, 0, g.T, scale, static_cast<const float *>(q),
                        static_cast<const float *>(k), static_cast<const float *>(v), static_cast<float *>(o),
                        lse, st);
  }
  if (!d_supported(g.D)) return ST_ERR_UNSUPPORTED;
  if (g.T > 64) return ST_ERR_UNSUPPORTED;
  if (!st::is_aligned(q, 16) || !st::is_aligned(k, 16) || !st::is_aligned(v, 16) || !st::is_aligned(o, 16))
    return ST_ERR_ALIGN;
  if (!strides_aligned(g, 2)) return ST_ERR_ALIGN;
  return st::attn_temporal_bf16(g, lo, hi, scale, q, k, v, o, lse, desc->o_fp32, st);
}
