// Decoding at temperature T > 0: categorical draws from fp32 logits rows and the
// rejection-sampling consensus of one block (atlas summary "Limitations": sampling
// at T > 0 goes through rejection sampling). The consensus is standard speculative
// sampling (Leviathan et al. 2023; Chen et al. 2023):
//   q_i = softmax(draft row i / T), p_j = softmax(verify row j / T);
//   d_i is accepted iff u_i * q_{i-1}(d_i) < p_{i-1}(d_i), in order, up to the
//   first rejection (a = number accepted);
//   the last committed token is drawn with the uniform v from max(0, p_a - q_a)
//   when d_{a+1} was rejected, else from p_K.
// Every random number is an input uniform on [0, 1).
//
// A categorical draw from non-negative weights w_0..w_{V-1} with the uniform v is
// the inverse CDF: the first index j with w_j > 0 whose running sum exceeds v * Z.
// The running sums are taken in index order over tiles of 1024 elements, with one
// fixed fp32 evaluation order: inside a tile, element (j, lane) of sub-chunk j
// (32 consecutive elements) carries incl_j(lane) + S_{j-1}, where incl_j is the
// warp-inclusive scan of sub-chunk j and S the warp-inclusive scan of the 32
// sub-chunk totals; tile totals are that value at the tile's last element; the
// prefix over tiles is a sequential fp32 sum. The pass that finds the tile and
// the pass that finds the element recompute exactly the same fp32 values, so the
// element found lies in the tile found. Warps take whole tiles; the chosen tile is
// rescanned by one warp.
#pragma once

namespace orthrus {

constexpr int kSampThreads = 512;   // row statistics and the plan-free draws: one CTA per row
constexpr int kSampTile = 1024;     // elements of one CDF tile
constexpr int kSampMaxTiles = 256;  // vocab <= 262144

__device__ __forceinline__ float warp_incl_scan(float x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = __fadd_rn(x, y);
  }
  return x;
}

// Weights are given as a load of element k's logits (load) and the weight computed from them
// (value), so that a tile's loads can all be issued before any weight is computed.

// exp((z_k - m) / T): the unnormalised softmax weight at temperature T
struct TemperedWeight {
  const float* z;
  float m, inv_t;
  __device__ __forceinline__ float2 load(int k) const { return make_float2(z[k], 0.f); }
  __device__ __forceinline__ float value(float2 r) const { return expf(__fmul_rn(__fsub_rn(r.x, m), inv_t)); }
};

// max(0, p_k - q_k) with p = softmax(zv / T), q = softmax(zd / T) (row maxima and
// normalisers given)
struct ResidualWeight {
  const float* zv;
  const float* zd;
  float mv, md, inv_t, rzv, rzd;
  __device__ __forceinline__ float2 load(int k) const { return make_float2(zv[k], zd[k]); }
  __device__ __forceinline__ float value(float2 r) const {
    const float p = __fmul_rn(expf(__fmul_rn(__fsub_rn(r.x, mv), inv_t)), rzv);
    const float q = __fmul_rn(expf(__fmul_rn(__fsub_rn(r.y, md), inv_t)), rzd);
    return fmaxf(__fsub_rn(p, q), 0.f);
  }
};

// The 32 weights a lane holds in tile s: element s*1024 + j*32 + lane in x[j] (0 past V).
template <class W>
__device__ __forceinline__ void tile_load(const W& w, int s, int V, int lane, float (&x)[32]) {
  const int k0 = s * kSampTile + lane;
  if (s * kSampTile + kSampTile <= V) {  // a whole tile: every load issued first
    float2 r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = w.load(k0 + j * 32);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = w.value(r[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = k0 + j * 32 < V ? w.value(w.load(k0 + j * 32)) : 0.f;
  }
}

// Scanned sub-chunk totals of tile s (lane j: S_j) and the tile total (one warp).
template <class W>
__device__ __forceinline__ float tile_prepare(const W& w, int s, int V, int lane, float& S) {
  float x[32];
  tile_load(w, s, V, lane, x);
  float sub = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float t = __shfl_sync(0xffffffffu, warp_incl_scan(x[j], lane), 31);
    if (lane == j) sub = t;
  }
  S = warp_incl_scan(sub, lane);
  const float s31 = __shfl_sync(0xffffffffu, sub, 31);
  const float pre = __shfl_sync(0xffffffffu, S, 30);
  return __fadd_rn(s31, pre);  // the running value of the tile's last element
}

// First element of tile s with positive weight and base + running value > target,
// or -1 (one warp; S from tile_prepare of the same tile).
template <class W>
__device__ __forceinline__ int tile_find(const W& w, int s, int V, int lane, float S, float base, float target) {
  float x[32];
  tile_load(w, s, V, lane, x);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float incl = warp_incl_scan(x[j], lane);
    const float pre = __shfl_sync(0xffffffffu, S, j > 0 ? j - 1 : 0);
    const float r = j > 0 ? __fadd_rn(incl, pre) : incl;
    const unsigned bal = __ballot_sync(0xffffffffu, x[j] > 0.f && __fadd_rn(base, r) > target);
    if (bal) return s * kSampTile + j * 32 + __ffs((int)bal) - 1;
  }
  return -1;
}

// Last element of tile s with positive weight, or -1 (one warp).
template <class W>
__device__ __forceinline__ int tile_last_positive(const W& w, int s, int V, int lane) {
  float x[32];
  tile_load(w, s, V, lane, x);
#pragma unroll
  for (int j = 31; j >= 0; --j) {
    const unsigned bal = __ballot_sync(0xffffffffu, x[j] > 0.f);
    if (bal) return s * kSampTile + j * 32 + 31 - __clz((int)bal);
  }
  return -1;
}

struct SampleSmem {
  float tot[kSampMaxTiles];
  float run[kSampMaxTiles];
  float target;
  int sel, last;
};

// Inverse-CDF draw from the weights w(0..V-1) with the uniform v; the whole CTA (any
// multiple of 32 threads) calls it, and the result (or -1 when every weight is zero) is
// returned to every thread.
template <class W>
__device__ int sample_row(const W& w, int V, float v, SampleSmem& sm) {
  const int nt = (V + kSampTile - 1) / kSampTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int s = warp; s < nt; s += (int)(blockDim.x >> 5)) {
    float S;
    const float t = tile_prepare(w, s, V, lane, S);
    if (lane == 0) sm.tot[s] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float R = 0.f;
    for (int s = 0; s < nt; ++s) {
      R = __fadd_rn(R, sm.tot[s]);
      sm.run[s] = R;
    }
    const float target = __fmul_rn(v, R);
    int sel = -1;
    for (int s = 0; s < nt && sel < 0; ++s)
      if (sm.run[s] > target) sel = s;
    int last = -1;
    for (int s = nt - 1; s >= 0 && last < 0; --s)
      if (sm.tot[s] > 0.f) last = s;
    sm.target = target;
    sm.sel = sel;
    sm.last = last;
  }
  __syncthreads();
  __shared__ int result;
  if (warp == 0) {
    int r = -1;
    const int sel = sm.sel;
    if (sel >= 0) {
      float S;
      tile_prepare(w, sel, V, lane, S);
      r = tile_find(w, sel, V, lane, S, sel > 0 ? sm.run[sel - 1] : 0.f, sm.target);
      if (r < 0) r = tile_last_positive(w, sel, V, lane);  // crossing only at zero-weight elements
    } else if (sm.last >= 0) {
      r = tile_last_positive(w, sm.last, V, lane);  // v * Z rounded up to Z
    }
    if (lane == 0) result = r;
  }
  __syncthreads();
  const int r = result;
  __syncthreads();
  return r;
}

// One warp: the draw from the tile totals tot[0..nt) that tile_prepare gave for these weights.
// The same fp32 operations as sample_row (running sums from 0 in tile order, target = v * total,
// the rescan of the chosen tile), so the result is the same index. The totals are first copied
// to `stage` (shared memory, kSampMaxTiles floats) by the whole warp, so that lane 0's running
// sums read shared memory instead of waiting on one global load per tile.
template <class W>
__device__ int select_from_totals(const W& w, int V, float v, const float* tot_global, float* tot, int lane) {
  const int nt = (V + kSampTile - 1) / kSampTile;
  for (int s = lane; s < nt; s += 32) tot[s] = tot_global[s];
  __syncwarp();
  int sel = -1, last = -1;
  float base = 0.f, target = 0.f;
  if (lane == 0) {
    float R = 0.f;
    for (int s = 0; s < nt; ++s) R = __fadd_rn(R, tot[s]);
    target = __fmul_rn(v, R);
    float P = 0.f;
    for (int s = 0; s < nt; ++s) {
      const float Q = __fadd_rn(P, tot[s]);
      if (Q > target) {
        sel = s;
        base = P;
        break;
      }
      P = Q;
    }
    for (int s = nt - 1; s >= 0 && last < 0; --s)
      if (tot[s] > 0.f) last = s;
  }
  sel = __shfl_sync(0xffffffffu, sel, 0);
  last = __shfl_sync(0xffffffffu, last, 0);
  base = __shfl_sync(0xffffffffu, base, 0);
  target = __shfl_sync(0xffffffffu, target, 0);
  int r = -1;
  if (sel >= 0) {
    float S;
    tile_prepare(w, sel, V, lane, S);
    r = tile_find(w, sel, V, lane, S, base, target);
    if (r < 0) r = tile_last_positive(w, sel, V, lane);
  } else if (last >= 0) {
    r = tile_last_positive(w, last, V, lane);
  }
  return r;
}

struct RowStats {
  float m, s;
  bool bad;  // a NaN or +inf logit, or no finite one
};

// The CTA's maximum m of one row, then Z = sum exp((z - m) / T) (the second pass reads the row
// from L2). 16-byte loads when the row allows them.
__device__ RowStats row_max_sum(const float* z, int V, float inv_t) {
  __shared__ float red[32];
  __shared__ int any_bad;
  const bool vec = (V & 3) == 0 && ((uintptr_t)z & 15) == 0;
  const float4* z4 = reinterpret_cast<const float4*>(z);
  const int n4 = vec ? V / 4 : 0;
  float m = -INFINITY;
  bool bad = false;
#pragma unroll 4
  for (int k = threadIdx.x; k < n4; k += blockDim.x) {
    const float4 x = z4[k];
    bad |= !(x.x < INFINITY) | !(x.y < INFINITY) | !(x.z < INFINITY) | !(x.w < INFINITY);
    m = fmaxf(fmaxf(m, fmaxf(x.x, x.y)), fmaxf(x.z, x.w));
  }
  for (int k = 4 * n4 + threadIdx.x; k < V; k += blockDim.x) {
    const float x = z[k];
    bad |= !(x < INFINITY);
    m = fmaxf(m, x);
  }
  if (threadIdx.x == 0) any_bad = 0;
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if (bad) any_bad = 1;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
  RowStats r{m, 0.f, any_bad != 0 || m == -INFINITY};
  __syncthreads();
  if (r.bad) return r;
  float s = 0.f;
#pragma unroll 4
  for (int k = threadIdx.x; k < n4; k += blockDim.x) {
    const float4 x = z4[k];
    s += expf((x.x - m) * inv_t) + expf((x.y - m) * inv_t) + expf((x.z - m) * inv_t) + expf((x.w - m) * inv_t);
  }
  for (int k = 4 * n4 + threadIdx.x; k < V; k += blockDim.x) s += expf((z[k] - m) * inv_t);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  s = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  r.s = s;
  __syncthreads();
  return r;
}

// One categorical draw per row: out[r] ~ softmax(logits[r] / T) with uniforms[r], one CTA per
// row (the plan-free entry point). A NaN or +inf logit (or a row of -inf only) sets
// ORTHRUS_ERR_NAN and out[r] = -1.
__global__ void __launch_bounds__(kSampThreads) sample_rows_kernel(const float* logits, int V, float inv_t,
                                                                   const float* uniforms, int* out, int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ SampleSmem sm;
  const int row = blockIdx.x;
  const float* z = logits + (size_t)row * V;
  const RowStats st = row_max_sum(z, V, inv_t);  // only the maximum is used
  if (st.bad) {
    if (threadIdx.x == 0) {
      out[row] = -1;
      if (status) set_status(status, ORTHRUS_ERR_NAN);
    }
    return;
  }
  const int r = sample_row(TemperedWeight{z, st.m, inv_t}, V, uniforms[row], sm);
  if (threadIdx.x == 0) out[row] = r;
}

// ---- the decode step's split kernels (workspace: row statistics and tile totals) ----------
// For a step they run as: statistics of the draft rows, tile totals, draws (the drafts); after
// the verify view: statistics of the verify rows, consensus tile totals, consensus draw and
// commit. The split spreads each row's tiles over many CTAs; the draws are the same indices
// sample_rows_kernel and sample_row give.

constexpr int kTotThreads = 256;  // tile-totals CTA: 8 warps, one tile each
constexpr int kTotTiles = kTotThreads / 32;

// stats[r] = (max, sum exp((z - max) / T)) of rows: the first draft_rows from dl, the rest
// from vl. A row with a NaN or +inf logit, or only -inf, gets (NaN, 1) and sets ORTHRUS_ERR_NAN.
__global__ void __launch_bounds__(kSampThreads) row_stats_kernel(const float* dl, int draft_rows, const float* vl,
                                                                 int V, float inv_t, float2* stats, int* status) {
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x;
  const float* z = row < draft_rows ? dl + (size_t)row * V : vl + (size_t)(row - draft_rows) * V;
  const RowStats st = row_max_sum(z, V, inv_t);
  if (threadIdx.x == 0) {
    if (st.bad) {
      set_status(status, ORTHRUS_ERR_NAN);
      stats[row] = make_float2(NAN, 1.f);
    } else {
      stats[row] = make_float2(st.m, st.s);
    }
  }
}

// Tile totals of the draws from draft rows: grid (rows, ceil(tiles / 8)).
__global__ void __launch_bounds__(kTotThreads) draw_totals_kernel(const float* logits, int V, float inv_t,
                                                                  const float2* stats, float* tot) {
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x, lane = threadIdx.x & 31;
  const int s = blockIdx.y * kTotTiles + (threadIdx.x >> 5);
  const float m = stats[row].x;
  if (s >= (V + kSampTile - 1) / kSampTile || m != m) return;
  float S;
  const float t = tile_prepare(TemperedWeight{logits + (size_t)row * V, m, inv_t}, s, V, lane, S);
  if (lane == 0) tot[(size_t)row * kSampMaxTiles + s] = t;
}

// The draws: one warp per row; out[r] = -1 for a row flagged by row_stats_kernel.
__global__ void __launch_bounds__(32) draw_select_kernel(const float* logits, int V, float inv_t,
                                                         const float2* stats, const float* tot,
                                                         const float* uniforms, int* out) {
  griddep_wait();
  griddep_launch();
  __shared__ float stage[kSampMaxTiles];
  const int row = blockIdx.x, lane = threadIdx.x;
  const float m = stats[row].x;
  int r = -1;
  if (m == m)
    r = select_from_totals(TemperedWeight{logits + (size_t)row * V, m, inv_t}, V, uniforms[row],
                           tot + (size_t)row * kSampMaxTiles, stage, lane);
  if (lane == 0) out[row] = r;
}

struct ConsensusArgs {
  int* pending;
  const int* draft;     // [B][K]
  const float* dl;      // [B][K][V]
  const float* vl;      // [B][K+1][V]
  const float2* stats;  // draft rows [B*K], then verify rows [B*(K+1)]
  float* tot;           // [B][kSampMaxTiles]
  const float* u_acc;   // [B][K]
  const float* u_fin;   // [B]
  int *accept_len, *committed, *len, *status;
  int B, K, V;
  float inv_t;
};

// a for sequence b: the accept tests u * q < p in order, up to the first rejection. Threads
// 0..63 of the CTA take part; every CTA of the sequence computes the same a.
__device__ int consensus_accept_len(const ConsensusArgs& c, int b, unsigned* masks) {
  const int t = threadIdx.x, K = c.K, V = c.V;
  bool acc = false;
  if (t < K) {
    const int d = c.draft[b * K + t];
    if (d < 0 || d >= V) {
      set_status(c.status, ORTHRUS_ERR_ARG);
    } else {
      const float2 sd = c.stats[b * K + t];
      const float2 sv = c.stats[c.B * K + b * (K + 1) + t];
      const float eq = expf(__fmul_rn(__fsub_rn(c.dl[((size_t)b * K + t) * V + d], sd.x), c.inv_t));
      const float ep = expf(__fmul_rn(__fsub_rn(c.vl[((size_t)b * (K + 1) + t) * V + d], sv.x), c.inv_t));
      // u * q < p with q = eq / Zd, p = ep / Zv
      acc = __fmul_rn(__fmul_rn(c.u_acc[b * K + t], eq), sv.y) < __fmul_rn(ep, sd.y);
    }
  }
  if (t < 64) {
    const unsigned bal = __ballot_sync(0xffffffffu, acc);
    if ((t & 31) == 0) masks[t >> 5] = bal;
  }
  __syncthreads();
  const unsigned long long all = (unsigned long long)masks[0] | ((unsigned long long)masks[1] << 32);
  int a = __ffsll((long long)~all) - 1;  // first rejected draft
  if (a < 0 || a > c.K) a = c.K;
  return a;
}

__device__ __forceinline__ ResidualWeight residual_weight(const ConsensusArgs& c, int b, int a) {
  const size_t vrow = (size_t)b * (c.K + 1) + a;
  const float2 sv = c.stats[c.B * c.K + vrow], sd = c.stats[b * c.K + a];
  return ResidualWeight{c.vl + vrow * c.V, c.dl + ((size_t)b * c.K + a) * c.V, sv.x, sd.x, c.inv_t, 1.f / sv.y,
                        1.f / sd.y};
}

__device__ __forceinline__ TemperedWeight verify_weight(const ConsensusArgs& c, int b, int a) {
  const size_t vrow = (size_t)b * (c.K + 1) + a;
  return TemperedWeight{c.vl + vrow * c.V, c.stats[c.B * c.K + vrow].x, c.inv_t};
}

// Tile totals of the last token's weights (the residual after a rejection, else p_K):
// grid (B, ceil(tiles / 8)).
__global__ void __launch_bounds__(kTotThreads) consensus_totals_kernel(const ConsensusArgs c) {
  griddep_wait();
  griddep_launch();
  __shared__ unsigned masks[2];
  const int b = blockIdx.x, lane = threadIdx.x & 31;
  const int a = consensus_accept_len(c, b, masks);
  const int s = blockIdx.y * kTotTiles + (threadIdx.x >> 5);
  if (s >= (c.V + kSampTile - 1) / kSampTile) return;
  float S, t;
  if (a < c.K) t = tile_prepare(residual_weight(c, b, a), s, c.V, lane, S);
  else t = tile_prepare(verify_weight(c, b, a), s, c.V, lane, S);
  if (lane == 0) c.tot[(size_t)b * kSampMaxTiles + s] = t;
}

// The last token's draw and the commit, one CTA per sequence: committed[b] = d_1..d_a, last,
// then -1; accept_len[b] = a; pending[b] = last; len[b] += a + 1. With the status word set (by
// this step or earlier) nothing is committed: accept_len = -1, committed = -1.
__global__ void __launch_bounds__(kTotThreads) consensus_select_kernel(const ConsensusArgs c) {
  griddep_wait();
  griddep_launch();
  __shared__ SampleSmem sm;
  __shared__ unsigned masks[2];
  __shared__ int last_s;
  __shared__ float stage[kSampMaxTiles];
  const int b = blockIdx.x, t = threadIdx.x, K = c.K;
  const int a = consensus_accept_len(c, b, masks);
  if (t < 32) {
    const float* tot = c.tot + (size_t)b * kSampMaxTiles;
    const int r = a < K ? select_from_totals(residual_weight(c, b, a), c.V, c.u_fin[b], tot, stage, t)
                        : select_from_totals(verify_weight(c, b, a), c.V, c.u_fin[b], tot, stage, t);
    if (t == 0) last_s = r;
  }
  __syncthreads();
  int last = last_s;
  if (last < 0)  // the residual rounded to zero everywhere: draw from p_a
    last = sample_row(verify_weight(c, b, a), c.V, c.u_fin[b], sm);
  const bool err = *(volatile const int*)c.status != 0 || last < 0;
  if (t <= K) {
    int v;
    if (err) v = -1;
    else if (t < a) v = c.draft[b * K + t];
    else if (t == a) v = last;
    else v = -1;
    c.committed[b * (K + 1) + t] = v;
  }
  if (t == 0) {
    if (err) {
      c.accept_len[b] = -1;
    } else {
      c.accept_len[b] = a;
      c.pending[b] = last;
      c.len[b] += a + 1;
    }
  }
}

}  // namespace orthrus
