// V-Major selective communication (CoCoDiff article, "V-Major" section):
// per-token L1 change of V against the previous step, threshold mask, the
// ascending list of active tokens, and the cache update for active tokens.
//
// Design.  vmajor_mask_compact is two launches and no atomics, so its output
// is deterministic (vmajor_mask_compact_scatter is the same two launches, the
// first also copying the rows of every active token into the caches):
//   1. l1_mask: a warp streams the [C] rows of two tokens at a time with
//      16-byte loads (all of a lane's loads issued before any arithmetic), accumulates
//      |cur - prev| in fp32, reduces over the warp with a fixed butterfly
//      order, writes the mask byte, and each CTA writes the number of active
//      tokens of its tile of TILE tokens to the workspace.
//   2. compact: one CTA per 2048 tokens sums the counts of the L1 tiles
//      before it (an exclusive prefix read straight from the workspace),
//      ranks its active tokens with warp ballots and writes their indices in
//      ascending order; the last CTA also writes the total count.
// The read of 2 * N * C elements dominates; everything else is O(N).
#include "common.cuh"

namespace {

constexpr int TILE = 32;          // tokens per CTA of the L1 pass (8 warps x 4 tokens)
constexpr int THREADS = 256;
constexpr int VMAX = 12;          // 16-byte vectors per lane per tensor in flight
constexpr int CTILE = 2048;       // tokens per CTA of the compaction pass
constexpr int ROUNDS = CTILE / THREADS;  // 32-token ballots per warp

// One warp per active row: copies each tensor's row to its cache (and to the
// packed message buffer when present).  The (tensor, vector) pairs of a row
// are enumerated together and a lane loads NB of them before storing any, so
// the copy of a row costs one memory round trip, not one per vector.
struct ScatterArgs {
  const char *src[8];
  char *dst[8];
  char *packed[8];
};

// The warp copies row `row` of every tensor (16-byte vectors, rv per row):
// the (tensor, vector) pairs are enumerated together and a lane loads NB of
// them before storing any, so a row costs one memory round trip.
__device__ __forceinline__ void copy_row_warp(const ScatterArgs &a, int n_tensors, long long row, int rv,
                                              const st::FastDiv &frv, long long packed_row, int lane) {
  constexpr int NB = 10;
  const long long row_bytes = (long long)rv * 16;
  const int total = rv * n_tensors;
  for (int j0 = 0; j0 < total; j0 += 32 * NB) {
    uint4 v[NB];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < total) {
        const int t = int(st::fdiv(uint32_t(j), frv)), k = j - t * rv;
        // after_wait: this kernel may start before the one that wrote src has finished
        v[u] = __ldg(reinterpret_cast<const uint4 *>(st::after_wait(a.src[t]) + row * row_bytes) + k);
      }
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < total) {
        const int t = int(st::fdiv(uint32_t(j), frv)), k = j - t * rv;
        reinterpret_cast<uint4 *>(a.dst[t] + row * row_bytes)[k] = v[u];
        if (packed_row >= 0 && a.packed[t]) reinterpret_cast<uint4 *>(a.packed[t] + packed_row * row_bytes)[k] = v[u];
      }
    }
  }
}

// SCATTER: the warp that decides a token is active also copies its rows of
// the scatter tensors into their caches (the fused mask + cache update).
template <typename T, bool SCATTER = false>
__global__ void __launch_bounds__(THREADS, 2) l1_mask(const char *__restrict__ cur,
                                                   const char *__restrict__ prev, long long n,
                                                   int row_vecs, float tau, int force_all,
                                                   unsigned char *__restrict__ mask,
                                                   float *__restrict__ l1_out,
                                                   int *__restrict__ tile_count, ScatterArgs sa = ScatterArgs{},
                                                   int n_tensors = 0, int scatter_vecs = 0,
                                                   st::FastDiv frv = st::FastDiv{1, 1u << 31, 31}) {
  constexpr int EPV = 16 / int(sizeof(T));
  constexpr int TPW = SCATTER ? 1 : 2;           // tokens of a warp in flight together
  constexpr int VM = VMAX / 2;                   // vectors per lane per token per tensor in flight
  __shared__ int warp_cnt[THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  cur = st::after_wait(cur);
  prev = st::after_wait(prev);
  int active = 0;
  for (int r = warp; r < TILE; r += TPW * (THREADS / 32)) {
    long long tok[TPW];
    float acc[TPW];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      tok[i] = (long long)blockIdx.x * TILE + r + i * (THREADS / 32);
      acc[i] = 0.f;
    }
    for (int v0 = 0; v0 < row_vecs; v0 += 32 * VM) {
      uint4 va[TPW][VM], vb[TPW][VM];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const uint4 *a = reinterpret_cast<const uint4 *>(cur) + tok[i] * row_vecs;
        const uint4 *b = reinterpret_cast<const uint4 *>(prev) + tok[i] * row_vecs;
#pragma unroll
        for (int u = 0; u < VM; ++u) {
          const int v = v0 + u * 32 + lane;
          if (tok[i] < n && v < row_vecs) { va[i][u] = __ldg(a + v); vb[i][u] = __ldg(b + v); }
        }
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
#pragma unroll
        for (int u = 0; u < VM; ++u) {
          const int v = v0 + u * 32 + lane;
          if (tok[i] < n && v < row_vecs) {
#pragma unroll
            for (int k = 0; k < EPV; ++k) {
              float x, y;
              if constexpr (sizeof(T) == 2) {
                x = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&va[i][u])[k]);
                y = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&vb[i][u])[k]);
              } else {
                x = reinterpret_cast<const float *>(&va[i][u])[k];
                y = reinterpret_cast<const float *>(&vb[i][u])[k];
              }
              acc[i] += fabsf(x - y);
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
      if (tok[i] < n) {
        const int m = (force_all || acc[i] > tau) ? 1 : 0;   // the same on every lane (butterfly sum)
        if (lane == 0) {
          mask[tok[i]] = (unsigned char)m;
          if (l1_out) l1_out[tok[i]] = acc[i];
        }
        active += m;
        if (SCATTER && m) copy_row_warp(sa, n_tensors, tok[i], scatter_vecs, frv, -1, lane);
      }
    }
  }
  if (lane == 0) warp_cnt[warp] = active;
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < THREADS / 32; ++w) c += warp_cnt[w];
    tile_count[blockIdx.x] = c;
  }
}

// The fused mask + cache update when the current V is itself one of the
// tensors whose rows are cached (the V-Major step: the caches of K and V take
// the active tokens' rows of this step's K and V) and a row is at most 32 * RV
// vectors: the warp loads the token's whole current and previous rows at once
// (one memory round trip), takes the L1 sum in l1_mask's order (same bits),
// and an active token's current row goes into its cache straight from the
// registers that hold it; the rows of the other tensors are copied with all
// of a lane's loads issued before its stores (one more round trip).  The two
// rows in flight per lane take about 100 registers: one CTA (eight warps) per
// SM, each warp with 12 KB of loads in flight (measured: 0.103 ms at 20736
// tokens of 3072 channels and half of them active, against 0.109 ms for
// l1_mask's scatter path; with the previous row in two halves, two CTAs per
// SM spill registers).  keep: bit t set when src[t] is the current V.
template <typename T, int RV>
__global__ void __launch_bounds__(THREADS, 1) l1_mask_keep(const char *__restrict__ cur,
                                                        const char *__restrict__ prev, long long n, int row_vecs,
                                                        float tau, int force_all, unsigned char *__restrict__ mask,
                                                        float *__restrict__ l1_out, int *__restrict__ tile_count,
                                                        const __grid_constant__ ScatterArgs sa, int n_tensors,
                                                        unsigned keep) {
  constexpr int EPV = 16 / int(sizeof(T));
  __shared__ int warp_cnt[THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  cur = st::after_wait(cur);
  prev = st::after_wait(prev);
  const long long row_bytes = (long long)row_vecs * 16;
  int active = 0;
  for (int r = warp; r < TILE; r += THREADS / 32) {
    const long long tok = (long long)blockIdx.x * TILE + r;
    if (tok >= n) break;                              // the same for every lane of the warp
    const uint4 *a = reinterpret_cast<const uint4 *>(cur + tok * row_bytes);
    const uint4 *b = reinterpret_cast<const uint4 *>(prev + tok * row_bytes);
    uint4 vc[RV], vp[RV];
#pragma unroll
    for (int u = 0; u < RV; ++u) {
      const int v = u * 32 + lane;
      if (v < row_vecs) {
        vc[u] = __ldg(a + v);
        vp[u] = __ldg(b + v);
      }
    }
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < RV; ++u) {
      if (u * 32 + lane < row_vecs) {
#pragma unroll
        for (int k = 0; k < EPV; ++k) {
          float x, y;
          if constexpr (sizeof(T) == 2) {
            x = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&vc[u])[k]);
            y = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&vp[u])[k]);
          } else {
            x = reinterpret_cast<const float *>(&vc[u])[k];
            y = reinterpret_cast<const float *>(&vp[u])[k];
          }
          acc += fabsf(x - y);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const int m = (force_all || acc > tau) ? 1 : 0;   // the same on every lane (butterfly sum)
    if (lane == 0) {
      mask[tok] = (unsigned char)m;
      if (l1_out) l1_out[tok] = acc;
    }
    active += m;
    if (!m) continue;
    // the current row first, into every cache that takes it (its registers are
    // then free) ... (the argument arrays are indexed in the parameter space)
    for (int t = 0; t < n_tensors; ++t) {
      if (!((keep >> t) & 1u)) continue;
      uint4 *d = reinterpret_cast<uint4 *>(sa.dst[t] + tok * row_bytes);
#pragma unroll
      for (int u = 0; u < RV; ++u)
        if (u * 32 + lane < row_vecs) d[u * 32 + lane] = vc[u];
    }
    // ... then the other tensors' rows, all of a lane's loads before its stores
    for (int t = 0; t < n_tensors; ++t) {
      if ((keep >> t) & 1u) continue;
      uint4 *d = reinterpret_cast<uint4 *>(sa.dst[t] + tok * row_bytes);
      // after_wait: this kernel may start before the one that wrote src has finished
      const uint4 *sr = reinterpret_cast<const uint4 *>(st::after_wait(sa.src[t]) + tok * row_bytes);
      uint4 w[RV];
#pragma unroll
      for (int u = 0; u < RV; ++u)
        if (u * 32 + lane < row_vecs) w[u] = __ldg(sr + u * 32 + lane);
#pragma unroll
      for (int u = 0; u < RV; ++u)
        if (u * 32 + lane < row_vecs) d[u * 32 + lane] = w[u];
    }
  }
  if (lane == 0) warp_cnt[warp] = active;
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < THREADS / 32; ++w) c += warp_cnt[w];
    tile_count[blockIdx.x] = c;
  }
}

// One CTA per CTILE tokens.  Exclusive prefix = sum of the L1-pass counts of
// the tiles before this CTA's first token, then warp ballots rank the active
// tokens inside the CTA in ascending order.
__global__ void __launch_bounds__(THREADS) compact(const unsigned char *__restrict__ mask, long long n,
                                                   int n_ctas, const int *__restrict__ tile_count,
                                                   int *__restrict__ idx, int *__restrict__ count) {
  __shared__ int red[THREADS / 32];
  __shared__ int warp_tot[THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  mask = st::after_wait(mask);
  tile_count = st::after_wait(tile_count);
  const long long first_tile = (long long)blockIdx.x * (CTILE / TILE);
  int part = 0;
  for (long long t = threadIdx.x; t < first_tile; t += THREADS) part += tile_count[t];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) red[warp] = part;
  // each warp owns ROUNDS consecutive groups of 32 tokens
  const long long tok0 = (long long)blockIdx.x * CTILE + (long long)warp * (ROUNDS * 32);
  unsigned bal[ROUNDS];
  int tot = 0;
#pragma unroll
  for (int r = 0; r < ROUNDS; ++r) {
    const long long tok = tok0 + r * 32 + lane;
    const int m = (tok < n) ? mask[tok] : 0;
    bal[r] = __ballot_sync(0xffffffffu, m);
    tot += __popc(bal[r]);
  }
  if (lane == 0) warp_tot[warp] = tot;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < THREADS / 32; ++w) base += red[w];
  int total_cta = 0;
  for (int w = 0; w < THREADS / 32; ++w) {
    if (w < warp) base += warp_tot[w];
    total_cta += warp_tot[w];
  }
#pragma unroll
  for (int r = 0; r < ROUNDS; ++r) {
    if ((bal[r] >> lane) & 1u) idx[base + __popc(bal[r] & ((1u << lane) - 1u))] = int(tok0 + r * 32 + lane);
    base += __popc(bal[r]);
  }
  if (blockIdx.x == n_ctas - 1 && threadIdx.x == 0) {
    int all = 0;
    for (int w = 0; w < THREADS / 32; ++w) all += red[w];
    *count = all + total_cta;
  }
}

__global__ void __launch_bounds__(256) scatter_rows(const int *__restrict__ idx,
                                                    const int *__restrict__ count, long long n,
                                                    long long row_bytes, int vec, int n_tensors,
                                                    ScatterArgs a, st::FastDiv frv) {
  st::pdl_trigger();
  st::pdl_wait();
  idx = st::after_wait(idx);
  count = st::after_wait(count);
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long cnt = *count;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long i = w; i < cnt && i < n; i += n_warps) {
    const long long row = idx[i];
    if (row < 0 || row >= n) continue;
    if (vec == 16) {
      copy_row_warp(a, n_tensors, row, int(row_bytes / 16), frv, i, lane);
    } else {
      for (int t = 0; t < n_tensors; ++t) {
        const char *s = a.src[t] + row * row_bytes;
        char *d = a.dst[t] + row * row_bytes;
        char *p = a.packed[t] ? a.packed[t] + i * row_bytes : nullptr;
        for (long long k = lane; k < row_bytes; k += 32) {
          const char v = s[k];
          d[k] = v;
          if (p) p[k] = v;
        }
      }
    }
  }
}

inline long long n_tiles_of(long long n) { return (n + TILE - 1) / TILE; }

// ---------------------------------------------------------------- sender-side V-Major
// V-Major decides on the sending side which tokens take part in the
// all-to-all [CC "V-Major"]: the change of V is measured on the spatially
// sharded layout x, and only the rows of active tokens move to their place in
// the temporally sharded layout y -- straight into the K/V caches that the
// attention reads.  Rows are enumerated in y order, so mask, per-tile counts
// and the compaction come out in y numbering.

// Destination row r of the S->T exchange -> its source row (the relayout
// formulas of ulysses_relayout, for one row): r = (q, b, i, j, t2, s2) in y,
// s2 = p * S/(N_S P) + s1, source (p, b, i, j, q * T/(N_T P) + t2, s1) in x.
struct RowMap {
  st::FastDiv fSs, fTq, fns, fnt, fB, fSp;
  int Ss, Tq, n_s, n_t, B, Sp, Tn;
};

// y row -> x row; optionally s1 (the row's index in its x segment of Sp
// rows) and pos (the token's index s in its frame, j * Ss + s2).
__device__ __forceinline__ long long y_to_x(const RowMap &m, long long r, int *s1_out = nullptr,
                                            int *pos_out = nullptr) {
  uint32_t g = uint32_t(r);                    // rows < 2^31 (checked on the host)
  const uint32_t rest = st::fdiv(g, m.fSs), s2 = g - rest * m.Ss;
  const uint32_t blk = st::fdiv(rest, m.fTq), t2 = rest - blk * m.Tq;
  const uint32_t b2 = st::fdiv(blk, m.fns), j = blk - b2 * m.n_s;
  const uint32_t qb = st::fdiv(b2, m.fnt), i = b2 - qb * m.n_t;
  const uint32_t q = st::fdiv(qb, m.fB), b = qb - q * m.B;
  const uint32_t p = st::fdiv(s2, m.fSp), s1 = s2 - p * m.Sp;
  if (s1_out) *s1_out = int(s1);
  if (pos_out) *pos_out = int(j * m.Ss + s2);
  const long long blk_x = (((long long)p * m.B + b) * m.n_t + i) * m.n_s + j;
  return (blk_x * m.Tn + (long long)q * m.Tq + t2) * m.Sp + s1;
}

// l1_mask over destination rows: the current and previous V rows are read at
// the source (x) row, the L1 change decides the mask of the destination row,
// and an active row is stored into the V cache at the destination -- from the
// registers that hold it when the row fits one pass of the warp, else read
// again.
template <typename T>
__global__ void __launch_bounds__(THREADS, 2) l1_relayout(const char *__restrict__ cur, const char *__restrict__ prev,
                                                       char *__restrict__ cache, long long n, int row_vecs,
                                                       float tau, int force_all, unsigned char *__restrict__ mask,
                                                       float *__restrict__ l1_out, int *__restrict__ tile_count,
                                                       RowMap rm) {
  constexpr int EPV = 16 / int(sizeof(T));
  constexpr int TPW = 2;
  constexpr int VM = 5;                          // 160 vectors per pass: a 1152-channel bf16 row in one
  __shared__ int warp_cnt[THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  cur = st::after_wait(cur);
  prev = st::after_wait(prev);
  const bool one_pass = row_vecs <= 32 * VM;
  int active = 0;
  for (int r = warp; r < TILE; r += TPW * (THREADS / 32)) {
    long long tok[TPW], src[TPW];
    float acc[TPW];
    uint4 va[TPW][VM];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      tok[i] = (long long)blockIdx.x * TILE + r + i * (THREADS / 32);
      src[i] = tok[i] < n ? y_to_x(rm, tok[i]) : 0;
      acc[i] = 0.f;
    }
    for (int v0 = 0; v0 < row_vecs; v0 += 32 * VM) {
      uint4 vb[TPW][VM];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const uint4 *a = reinterpret_cast<const uint4 *>(cur) + src[i] * row_vecs;
        const uint4 *b = reinterpret_cast<const uint4 *>(prev) + src[i] * row_vecs;
#pragma unroll
        for (int u = 0; u < VM; ++u) {
          const int v = v0 + u * 32 + lane;
          if (tok[i] < n && v < row_vecs) { va[i][u] = __ldg(a + v); vb[i][u] = __ldg(b + v); }
        }
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
#pragma unroll
        for (int u = 0; u < VM; ++u) {
          const int v = v0 + u * 32 + lane;
          if (tok[i] < n && v < row_vecs) {
#pragma unroll
            for (int k = 0; k < EPV; ++k) {
              float x, y;
              if constexpr (sizeof(T) == 2) {
                x = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&va[i][u])[k]);
                y = st::bf16_to_f32(reinterpret_cast<const uint16_t *>(&vb[i][u])[k]);
              } else {
                x = reinterpret_cast<const float *>(&va[i][u])[k];
                y = reinterpret_cast<const float *>(&vb[i][u])[k];
              }
              acc[i] += fabsf(x - y);
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
      if (tok[i] < n) {
        const int m = (force_all || acc[i] > tau) ? 1 : 0;   // the same on every lane (butterfly sum)
        if (lane == 0) {
          mask[tok[i]] = (unsigned char)m;
          if (l1_out) l1_out[tok[i]] = acc[i];
        }
        active += m;
        if (m) {
          uint4 *d = reinterpret_cast<uint4 *>(cache) + tok[i] * row_vecs;
          if (one_pass) {
#pragma unroll
            for (int u = 0; u < VM; ++u) {
              const int v = u * 32 + lane;
              if (v < row_vecs) d[v] = va[i][u];
            }
          } else {
            const uint4 *a = reinterpret_cast<const uint4 *>(cur) + src[i] * row_vecs;
            for (int v = lane; v < row_vecs; v += 32) d[v] = __ldg(a + v);
          }
        }
      }
    }
  }
  if (lane == 0) warp_cnt[warp] = active;
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < THREADS / 32; ++w) c += warp_cnt[w];
    tile_count[blockIdx.x] = c;
  }
}

// The S->T move of the rows listed in idx[0, *count) without the RMSNorm: a
// warp copies one listed row with 16-byte vectors.
__global__ void __launch_bounds__(256) rows_idx(const char *__restrict__ in, char *__restrict__ out,
                                                const int *__restrict__ idx, const int *__restrict__ count,
                                                long long n, int row_vecs, RowMap rm) {
  const int lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  in = st::after_wait(in);
  idx = st::after_wait(idx);
  count = st::after_wait(count);
  const long long n_act = min(max((long long)*count, 0LL), n);   // a listed row outside [0, n) is skipped
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long k = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; k < n_act; k += nw) {
    const long long r = idx[k];
    if (r < 0 || r >= n) continue;
    const uint4 *a = reinterpret_cast<const uint4 *>(in) + y_to_x(rm, r) * row_vecs;
    uint4 *d = reinterpret_cast<uint4 *>(out) + r * row_vecs;
    for (int v = lane; v < row_vecs; v += 32) d[v] = __ldg(a + v);
  }
}

__device__ unsigned int g_vmajor_error;      // bounded waits of the gather kernel that ran out
constexpr unsigned long long VM_WAIT_NS = 2000000000ull;   // 2 s per wait
constexpr int GATHER_WARPS = 4;

__device__ __forceinline__ uint32_t sh_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// The S->T move of the rows listed in idx[0, *count) (K of the active tokens
// into the K cache), with the per-head RMSNorm of ulysses_relayout computed in
// the same order (same bytes).  A warp task is the RPT listed rows whose heads
// fill a 32-head buffer; the bulk copy engine brings each row in (one copy per
// row) while the previous task is normalised, one lane normalises one head in
// shared memory, and one bulk copy per row writes it back.
// Five CTAs per SM (20 warps) without the rotation: registers capped for it,
// and the launch asks for the largest shared-memory carveout.
template <typename T, int D, bool ROPE>
__global__ void __launch_bounds__(GATHER_WARPS * 32, ROPE ? 1 : 5) rows_gather_rms(const char *__restrict__ in, char *__restrict__ out,
                                                                     const int *__restrict__ idx,
                                                                     const int *__restrict__ count, long long n,
                                                                     int row_vecs, const float *__restrict__ gamma,
                                                                     float eps, RowMap rm,
                                                                     const float2 *__restrict__ rope) {
  constexpr int EPV = 16 / int(sizeof(T));
  constexpr int VPH = D / EPV;                 // vectors per head
  constexpr int HB = D * int(sizeof(T));       // bytes per head
  constexpr int BUF = 32 * HB;
  constexpr int ROT = VPH % 4 == 0 ? 1 : 0;    // the full relayout's per-lane rotation of the vector order
  extern __shared__ __align__(128) uint8_t rg_smem[];
  __shared__ __align__(8) uint64_t full[GATHER_WARPS][2];
  __shared__ float g_s[D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st::pdl_trigger();
  st::pdl_wait();
  in = st::after_wait(in);
  idx = st::after_wait(idx);
  count = st::after_wait(count);
  gamma = st::after_wait(gamma);
  if constexpr (ROPE) rope = st::after_wait(rope);
  for (int d = threadIdx.x; d < D; d += blockDim.x) g_s[d] = gamma[d];
  if (lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sh_u32(&full[warp][0])) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sh_u32(&full[warp][1])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int row_bytes = row_vecs * 16;
  const int hpr = row_bytes / HB;              // heads per row (<= 32)
  const int rpt = 32 / hpr;                    // rows per task
  const long long n_act = min(max((long long)*count, 0LL), n);   // a listed row outside [0, n) is skipped
  const long long n_tasks = (n_act + rpt - 1) / rpt;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  uint8_t *buf0 = rg_smem + warp * 2 * BUF;
  // lane 0: load the rows of task t into buffer b; returns the rows in range as bits
  auto issue = [&](long long t, int b) -> uint32_t {
    const int nr = int(min((long long)rpt, n_act - t * rpt));
    uint32_t vm = 0;
    for (int j = 0; j < nr; ++j) {
      const int r = idx[t * rpt + j];
      if (r >= 0 && r < n) vm |= 1u << j;
    }
    uint64_t *bar = &full[warp][b];
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sh_u32(bar)),
                 "r"(uint32_t(__popc(vm)) * uint32_t(row_bytes))
                 : "memory");
    for (int j = 0; j < nr; ++j) {
      if (!((vm >> j) & 1u)) continue;
      const long long src = y_to_x(rm, idx[t * rpt + j]);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(sh_u32(buf0 + b * BUF + j * row_bytes)), "l"(in + src * row_bytes), "r"(row_bytes),
                   "r"(sh_u32(bar))
                   : "memory");
    }
    return vm;
  };
  bool ok = true;
  uint32_t vm_cur = 0, vm_next = 0;             // bit j: row j of the task is in range and moves
  if (lane == 0 && gw < n_tasks) vm_cur = issue(gw, 0);
  vm_cur = __shfl_sync(0xffffffffu, vm_cur, 0);
  int i = 0;
  for (long long t = gw; t < n_tasks && ok; t += nw, ++i) {
    const int b = i & 1;
    const long long next = t + nw;
    if (next < n_tasks) {
      if (lane == 0) {
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // the other buffer's stores have read it
        vm_next = issue(next, b ^ 1);
      }
      vm_next = __shfl_sync(0xffffffffu, vm_next, 0);
    }
    if (lane == 0) {
      const unsigned long long t0 = gtimer();
      uint32_t done = 0;
      while (!done) {
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}\n"
                     : "=r"(done) : "r"(sh_u32(&full[warp][b])), "r"(uint32_t((i >> 1) & 1)) : "memory");
        if (!done && gtimer() - t0 > VM_WAIT_NS) {
          atomicOr(&g_vmajor_error, 1u);
          ok = false;
          break;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    uint8_t *bufp = buf0 + b * BUF;
    if (lane < rpt * hpr && ((vm_cur >> (lane / hpr)) & 1u)) {
      const int j = lane / hpr, h = lane - j * hpr;
      // the full relayout normalises head (s1 * hpr + h) of a segment on lane (s1 * hpr + h) % 32
      int s1, pos = 0;
      y_to_x(rm, idx[t * rpt + j], &s1, ROPE ? &pos : nullptr);
      const int fl = (s1 * hpr + h) % 32;
      const int r0 = (fl * ROT) % VPH;
      auto uix = [&](int u0) { return u0 + r0 < VPH ? u0 + r0 : u0 + r0 - VPH; };
      uint8_t *hp = bufp + j * row_bytes + h * HB;
      // rotary angles of the row's token (its index s in the frame); the first
      // group of pairs is on its way during the sum of squares
      const float2 *rot = ROPE ? rope + (long long)pos * (D / 2) : nullptr;
      st::RotVec<T> cs[st::RG];
      if constexpr (ROPE) {
#pragma unroll
        for (int g = 0; g < st::RG && g < VPH; ++g) cs[g] = st::load_rot<T>(rot + uix(g) * (EPV / 2));
      }
      float ss = 0.f;
#pragma unroll
      for (int u0 = 0; u0 < VPH; ++u0) {
        const int u = uix(u0);
        const uint4 v = *reinterpret_cast<const uint4 *>(hp + u * 16);
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
        const uint4 v = *reinterpret_cast<const uint4 *>(hp + u * 16);
        *reinterpret_cast<uint4 *>(hp + u * 16) = st::rms_rope_vec<T, ROPE>(v, inv, g_s + u * EPV, cs[u0 % st::RG]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      for (int j = 0; j < rpt; ++j)
        if ((vm_cur >> j) & 1u)
          asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                     ::"l"(out + (long long)idx[t * rpt + j] * row_bytes), "r"(sh_u32(bufp + j * row_bytes)),
                     "r"(row_bytes)
                     : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    vm_cur = vm_next;
  }
  if (lane == 0) {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    if (!ok) {
      // the next task's rows may still be landing in the other buffer: wait for them (bounded)
      const unsigned long long t0 = gtimer();
      uint32_t done = 0;
      while (!done && gtimer() - t0 < VM_WAIT_NS)
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}\n"
                     : "=r"(done) : "r"(sh_u32(&full[warp][(i + 1) & 1])), "r"(uint32_t(((i + 1) >> 1) & 1))
                     : "memory");
    }
  }
  __syncwarp();
}

template <typename T>
st_status launch_gather_rms(int D, const char *in, char *out, const int *idx, const int *count, long long n,
                            int row_vecs, const float *gamma, float eps, RowMap rm, cudaStream_t s,
                            const float2 *rope) {
#define ST_GATHER(DD)                                                                                       \
  {                                                                                                         \
    auto kern = rope ? rows_gather_rms<T, DD, true> : rows_gather_rms<T, DD, false>;                       \
    const int smem = GATHER_WARPS * 2 * 32 * DD * int(sizeof(T));                                           \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||     \
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)     \
      return ST_ERR_CUDA;                                                                                   \
    int per_sm = 0;                                                                                         \
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, GATHER_WARPS * 32, smem) != cudaSuccess || \
        per_sm < 1)                                                                                         \
      per_sm = 1;                                                                                           \
    const int hpr = row_vecs * 16 / (DD * int(sizeof(T)));                                                  \
    const long long tasks = (n + 32 / hpr - 1) / (32 / hpr); /* at most: every row listed */                \
    const long long want = (tasks + GATHER_WARPS - 1) / GATHER_WARPS;                                       \
    const long long cap = (long long)st::num_sms() * per_sm;                                                \
    const int grid = int(want < cap ? want : cap);                                                          \
    return st::launch_pdl(kern, grid, GATHER_WARPS * 32, smem, s, in, out, idx, count, n, row_vecs, gamma, eps, rm, \
                          rope);                                                                            \
  }
  switch (D) {
    case 32: ST_GATHER(32)
    case 64: ST_GATHER(64)
    case 72: ST_GATHER(72)
    case 80: ST_GATHER(80)
    case 96: ST_GATHER(96)
    case 128: ST_GATHER(128)
  }
#undef ST_GATHER
  return ST_ERR_UNSUPPORTED;
}

// Host-side check and map of the S->T exchange shape (elem: element bytes).
st_status make_rowmap(int P, int B, int T, int S, int C, int n_t, int n_s, int elem, RowMap &m, long long &rows) {
  if (P <= 0 || B <= 0 || T <= 0 || S <= 0 || C <= 0 || n_t <= 0 || n_s <= 0) return ST_ERR_SHAPE;
  if (T % (n_t * P) || S % (n_s * P)) return ST_ERR_DIVISIBILITY;
  if (((long long)C * elem) % 16) return ST_ERR_ALIGN;
  rows = (long long)B * T * S;
  if (rows >= (1LL << 31)) return ST_ERR_SHAPE;
  m.Ss = S / n_s;
  m.Tq = T / (n_t * P);
  m.n_s = n_s;
  m.n_t = n_t;
  m.B = B;
  m.Sp = S / (n_s * P);
  m.Tn = T / n_t;
  m.fSs = st::make_fastdiv(uint32_t(m.Ss));
  m.fTq = st::make_fastdiv(uint32_t(m.Tq));
  m.fns = st::make_fastdiv(uint32_t(n_s));
  m.fnt = st::make_fastdiv(uint32_t(n_t));
  m.fB = st::make_fastdiv(uint32_t(B));
  m.fSp = st::make_fastdiv(uint32_t(m.Sp));
  return ST_OK;
}

}  // namespace

ST_API size_t vmajor_workspace_bytes(long long n_tokens) {
  if (n_tokens <= 0) return 0;
  return size_t(n_tiles_of(n_tokens)) * sizeof(int);
}

ST_API st_status vmajor_mask_compact(const void *v_cur, const void *v_prev, long long n_tokens, int C,
                                     st_dtype dtype, float tau, int force_all, unsigned char *mask,
                                     int *idx, int *count, float *l1_out, void *workspace,
                                     size_t workspace_bytes, st_stream_t stream) {
  if (!v_cur || !v_prev || !mask || !idx || !count) return ST_ERR_NULL;
  if (n_tokens <= 0 || C <= 0 || n_tokens >= (1LL << 31)) return ST_ERR_SHAPE;
  if (dtype != ST_F32 && dtype != ST_BF16) return ST_ERR_DTYPE;
  const int esize = dtype == ST_F32 ? 4 : 2;
  if ((C * esize) % 16 || !st::is_aligned(v_cur, 16) || !st::is_aligned(v_prev, 16)) return ST_ERR_ALIGN;
  if (!workspace) return ST_ERR_NULL;
  if (workspace_bytes < vmajor_workspace_bytes(n_tokens)) return ST_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long tiles = n_tiles_of(n_tokens);
  if (tiles > 0x7fffffffLL) return ST_ERR_SHAPE;
  const int row_vecs = C * esize / 16;
  int *tile_count = static_cast<int *>(workspace);
  const char *cur = static_cast<const char *>(v_cur), *prev = static_cast<const char *>(v_prev);
  st_status st = dtype == ST_BF16
                     ? st::launch_pdl(l1_mask<uint16_t>, int(tiles), THREADS, 0, s, cur, prev, n_tokens, row_vecs,
                                      tau, force_all, mask, l1_out, tile_count, ScatterArgs{}, 0, 0, st::make_fastdiv(1))
                     : st::launch_pdl(l1_mask<float>, int(tiles), THREADS, 0, s, cur, prev, n_tokens, row_vecs, tau,
                                      force_all, mask, l1_out, tile_count, ScatterArgs{}, 0, 0, st::make_fastdiv(1));
  if (st != ST_OK) return st;
  const int ctas = int((n_tokens + CTILE - 1) / CTILE);
  return st::launch_pdl(compact, ctas, THREADS, 0, s, static_cast<const unsigned char *>(mask), n_tokens, ctas,
                        static_cast<const int *>(tile_count), idx, count);
}

ST_API st_status vmajor_mask_compact_scatter(const void *v_cur, const void *v_prev, long long n_tokens, int C,
                                             st_dtype dtype, float tau, int force_all, unsigned char *mask, int *idx,
                                             int *count, float *l1_out, void *workspace, size_t workspace_bytes,
                                             const void *const *src, void *const *dst_cache, int n_tensors,
                                             st_stream_t stream) {
  if (!v_cur || !v_prev || !mask || !idx || !count || !src || !dst_cache) return ST_ERR_NULL;
  if (n_tokens <= 0 || C <= 0 || n_tokens >= (1LL << 31)) return ST_ERR_SHAPE;
  if (n_tensors < 1 || n_tensors > 8) return ST_ERR_SHAPE;
  if (dtype != ST_F32 && dtype != ST_BF16) return ST_ERR_DTYPE;
  const int esize = dtype == ST_F32 ? 4 : 2;
  if ((C * esize) % 16 || !st::is_aligned(v_cur, 16) || !st::is_aligned(v_prev, 16)) return ST_ERR_ALIGN;
  if (!workspace) return ST_ERR_NULL;
  if (workspace_bytes < vmajor_workspace_bytes(n_tokens)) return ST_ERR_SHAPE;
  const int row_vecs = C * esize / 16;
  if ((long long)row_vecs * n_tensors >= (1LL << 31)) return ST_ERR_SHAPE;
  ScatterArgs a = {};
  for (int t = 0; t < n_tensors; ++t) {
    if (!src[t] || !dst_cache[t]) return ST_ERR_NULL;
    if (!st::is_aligned(src[t], 16) || !st::is_aligned(dst_cache[t], 16)) return ST_ERR_ALIGN;
    a.src[t] = static_cast<const char *>(src[t]);
    a.dst[t] = static_cast<char *>(dst_cache[t]);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long tiles = n_tiles_of(n_tokens);
  if (tiles > 0x7fffffffLL) return ST_ERR_SHAPE;
  int *tile_count = static_cast<int *>(workspace);
  const char *cur = static_cast<const char *>(v_cur), *prev = static_cast<const char *>(v_prev);
  unsigned keep = 0;                                   // scatter sources that are the current V itself
  for (int t = 0; t < n_tensors; ++t)
    if (src[t] == v_cur) keep |= 1u << t;
  constexpr int KEEP_RV = 12;                          // rows up to 32 * 12 vectors (C = 3072 in bf16)
  st_status st;
  if (keep && row_vecs <= 32 * KEEP_RV)
    st = dtype == ST_BF16 ? st::launch_pdl(l1_mask_keep<uint16_t, KEEP_RV>, int(tiles), THREADS, 0, s, cur, prev,
                                           n_tokens, row_vecs, tau, force_all, mask, l1_out, tile_count, a,
                                           n_tensors, keep)
                          : st::launch_pdl(l1_mask_keep<float, KEEP_RV>, int(tiles), THREADS, 0, s, cur, prev,
                                           n_tokens, row_vecs, tau, force_all, mask, l1_out, tile_count, a,
                                           n_tensors, keep);
  else
    st = dtype == ST_BF16
                     ? st::launch_pdl(l1_mask<uint16_t, true>, int(tiles), THREADS, 0, s, cur, prev, n_tokens,
                                      row_vecs, tau, force_all, mask, l1_out, tile_count, a, n_tensors, row_vecs,
                                      st::make_fastdiv(uint32_t(row_vecs)))
                     : st::launch_pdl(l1_mask<float, true>, int(tiles), THREADS, 0, s, cur, prev, n_tokens, row_vecs,
                                      tau, force_all, mask, l1_out, tile_count, a, n_tensors, row_vecs,
                                      st::make_fastdiv(uint32_t(row_vecs)));
  if (st != ST_OK) return st;
  const int ctas = int((n_tokens + CTILE - 1) / CTILE);
  return st::launch_pdl(compact, ctas, THREADS, 0, s, static_cast<const unsigned char *>(mask), n_tokens, ctas,
                        static_cast<const int *>(tile_count), idx, count);
}

ST_API st_status vmajor_scatter_rows(const int *idx, const int *count, long long n_tokens, int C,
                                     int elem_bytes, const void *const *src, void *const *dst_cache,
                                     int n_tensors, void *const *packed, st_stream_t stream) {
  if (!idx || !count || !src || !dst_cache) return ST_ERR_NULL;
  if (n_tensors < 1 || n_tensors > 8 || n_tokens <= 0 || C <= 0) return ST_ERR_SHAPE;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return ST_ERR_DTYPE;
  ScatterArgs a = {};
  const long long row_bytes = (long long)C * elem_bytes;
  bool all16 = (row_bytes % 16) == 0;
  for (int t = 0; t < n_tensors; ++t) {
    if (!src[t] || !dst_cache[t]) return ST_ERR_NULL;
    a.src[t] = static_cast<const char *>(src[t]);
    a.dst[t] = static_cast<char *>(dst_cache[t]);
    a.packed[t] = packed ? static_cast<char *>(packed[t]) : nullptr;
    all16 = all16 && st::is_aligned(src[t], 16) && st::is_aligned(dst_cache[t], 16) &&
            (!a.packed[t] || st::is_aligned(a.packed[t], 16));
  }
  if (all16 && (row_bytes / 16) * n_tensors >= (1LL << 31)) return ST_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long want = (n_tokens * 32 + 255) / 256;
  const long long cap = (long long)st::num_sms() * 16;
  const int grid = int(want < cap ? want : cap);
  return st::launch_pdl(scatter_rows, grid, 256, 0, s, idx, count, n_tokens, row_bytes, all16 ? 16 : 1, n_tensors,
                        a, st::make_fastdiv(uint32_t(all16 ? row_bytes / 16 : 1)));
}

// ---------------------------------------------------------------------------
// Allocation-free variant of vmajor_mask_compact.
//
// Some callers may not allocate device memory while they run: a serving loop
// that owns a fixed memory pool (or a budget fixed at start-up) must not grow
// it, and cudaMalloc can stall behind work in flight or fail under memory
// pressure at the worst moment.  This variant keeps its per-tile counts in a
// file-scope device array instead of a caller-provided workspace.  The array
// holds kStaticMaxTokens / TILE ints (512 KiB) on every GPU that loads the
// library, for the life of the process; larger inputs are rejected.
#include <mutex>

namespace {

constexpr long long kStaticMaxTokens = 1LL << 22;  // 4,194,304 tokens
constexpr long long kStaticTiles = kStaticMaxTokens / TILE;
__device__ __align__(256) int g_vmajor_static_counts[kStaticTiles];

// Device address of the array on the current device.  The first call on a
// device looks it up with that device current and caches it for the life of
// the process (so the entry point must not be used after a cudaDeviceReset of
// that device: the cached address would belong to the old context).
int *static_counts_on_current_device() {
  static std::mutex mu;
  static int *addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_vmajor_static_counts) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int *>(p);
  }
  return addr[dev];
}

}  // namespace

ST_API st_status vmajor_mask_compact_noalloc(const void *v_cur, const void *v_prev, long long n_tokens, int C,
                                             st_dtype dtype, float tau, int force_all, unsigned char *mask,
                                             int *idx, int *count, float *l1_out, st_stream_t stream) {
  if (!v_cur || !v_prev || !mask || !idx || !count) return ST_ERR_NULL;
  if (n_tokens <= 0 || C <= 0) return ST_ERR_SHAPE;
  if (n_tokens > kStaticMaxTokens) return ST_ERR_SHAPE;  // beyond the static scratch capacity
  if (dtype != ST_F32 && dtype != ST_BF16) return ST_ERR_DTYPE;
  const int esize = dtype == ST_F32 ? 4 : 2;
  if ((C * esize) % 16 || !st::is_aligned(v_cur, 16) || !st::is_aligned(v_prev, 16)) return ST_ERR_ALIGN;
  int *tile_count = static_counts_on_current_device();
  if (!tile_count) return ST_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long tiles = n_tiles_of(n_tokens);
  const int row_vecs = C * esize / 16;
  // every tile count is written by the first launch before the second reads
  // it, so nothing in the array has to start at zero
  if (dtype == ST_BF16)
    l1_mask<uint16_t><<<int(tiles), THREADS, 0, s>>>(static_cast<const char *>(v_cur),
                                                     static_cast<const char *>(v_prev), n_tokens, row_vecs, tau,
                                                     force_all, mask, l1_out, tile_count);
  else
    l1_mask<float><<<int(tiles), THREADS, 0, s>>>(static_cast<const char *>(v_cur),
                                                  static_cast<const char *>(v_prev), n_tokens, row_vecs, tau,
                                                  force_all, mask, l1_out, tile_count);
  st_status st = st::launch_status();
  if (st != ST_OK) return st;
  const int ctas = int((n_tokens + CTILE - 1) / CTILE);
  compact<<<ctas, THREADS, 0, s>>>(mask, n_tokens, ctas, tile_count, idx, count);
  return st::launch_status();
}

ST_API st_status vmajor_relayout_mask(const void *v_cur_x, const void *v_prev_x, void *v_cache_y, int P, int B, int T,
                                      int S, int C, int n_t, int n_s, st_dtype dtype, float tau, int force_all,
                                      unsigned char *mask, int *idx, int *count, float *l1_out, void *workspace,
                                      size_t workspace_bytes, st_stream_t stream) {
  if (!v_cur_x || !v_prev_x || !v_cache_y || !mask || !idx || !count || !workspace) return ST_ERR_NULL;
  if (dtype != ST_F32 && dtype != ST_BF16) return ST_ERR_DTYPE;
  const int esize = dtype == ST_F32 ? 4 : 2;
  RowMap rm;
  long long n = 0;
  st_status st = make_rowmap(P, B, T, S, C, n_t, n_s, esize, rm, n);
  if (st != ST_OK) return st;
  if (!st::is_aligned(v_cur_x, 16) || !st::is_aligned(v_prev_x, 16) || !st::is_aligned(v_cache_y, 16))
    return ST_ERR_ALIGN;
  if (workspace_bytes < vmajor_workspace_bytes(n)) return ST_ERR_SHAPE;
  const long long bytes = n * C * esize;
  const char *c0 = static_cast<const char *>(v_cur_x), *p0 = static_cast<const char *>(v_prev_x);
  char *d0 = static_cast<char *>(v_cache_y);
  if ((d0 < c0 + bytes && c0 < d0 + bytes) || (d0 < p0 + bytes && p0 < d0 + bytes)) return ST_ERR_SHAPE;  // overlap
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long tiles = n_tiles_of(n);
  const int row_vecs = C * esize / 16;
  int *tile_count = static_cast<int *>(workspace);
  st = dtype == ST_BF16
           ? st::launch_pdl(l1_relayout<uint16_t>, int(tiles), THREADS, 0, s, c0, p0, d0, n, row_vecs, tau,
                            force_all, mask, l1_out, tile_count, rm)
           : st::launch_pdl(l1_relayout<float>, int(tiles), THREADS, 0, s, c0, p0, d0, n, row_vecs, tau, force_all,
                            mask, l1_out, tile_count, rm);
  if (st != ST_OK) return st;
  const int ctas = int((n + CTILE - 1) / CTILE);
  return st::launch_pdl(compact, ctas, THREADS, 0, s, static_cast<const unsigned char *>(mask), n, ctas,
                        static_cast<const int *>(tile_count), idx, count);
}

ST_API st_status vmajor_relayout_rows(const void *in_x, void *out_y, const int *idx, const int *count, int P, int B,
                                      int T, int S, int C, int n_t, int n_s, st_dtype dtype, const float *rms_gamma,
                                      int rms_head_dim, float rms_eps, const float *rope_table, int rope_positions,
                                      st_stream_t stream) {
  if (!in_x || !out_y || !idx || !count) return ST_ERR_NULL;
  if (dtype != ST_F32 && dtype != ST_BF16) return ST_ERR_DTYPE;
  const int esize = dtype == ST_F32 ? 4 : 2;
  RowMap rm;
  long long n = 0;
  st_status st = make_rowmap(P, B, T, S, C, n_t, n_s, esize, rm, n);
  if (st != ST_OK) return st;
  if (!st::is_aligned(in_x, 16) || !st::is_aligned(out_y, 16)) return ST_ERR_ALIGN;
  const int row_vecs = C * esize / 16;
  if (rms_gamma) {
    if (rms_head_dim <= 0 || C % rms_head_dim || (rms_head_dim * esize) % 16) return ST_ERR_SHAPE;
    if (C / rms_head_dim > 32) return ST_ERR_UNSUPPORTED;     // a row's heads fill at most one task buffer
  }
  if (rope_table) {                                           // rides on the RMSNorm pass
    if (!rms_gamma) return ST_ERR_NULL;
    if (rms_head_dim % 2 || rope_positions < S) return ST_ERR_SHAPE;
    if (!st::is_aligned(rope_table, 16)) return ST_ERR_ALIGN;
  }
  const long long bytes = n * C * esize;
  const char *i0 = static_cast<const char *>(in_x);
  char *o0 = static_cast<char *>(out_y);
  if (o0 < i0 + bytes && i0 < o0 + bytes) return ST_ERR_SHAPE;  // overlap
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (rms_gamma)
    return dtype == ST_BF16 ? launch_gather_rms<uint16_t>(rms_head_dim, i0, o0, idx, count, n, row_vecs, rms_gamma,
                                                          rms_eps, rm, s, reinterpret_cast<const float2 *>(rope_table))
                            : launch_gather_rms<float>(rms_head_dim, i0, o0, idx, count, n, row_vecs, rms_gamma,
                                                       rms_eps, rm, s, reinterpret_cast<const float2 *>(rope_table));
  const long long want = (n + 7) / 8;
  const long long cap = (long long)st::num_sms() * 16;
  const int grid = int(want < cap ? want : cap);
  return st::launch_pdl(rows_idx, grid, 256, 0, s, i0, o0, idx, count, n, row_vecs, rm);
}

namespace st {
unsigned int read_and_clear_vmajor_error(cudaStream_t stream, cudaError_t *err) {
  unsigned int word = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&word, g_vmajor_error, sizeof(word), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_vmajor_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (err) *err = e;
  return word;
}
}  // namespace st
