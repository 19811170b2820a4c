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
// element found lies in the tile found. One CTA of 1024 threads per row; warps
// take tiles round-robin; the chosen tile is rescanned by warp 0.
#pragma once

namespace orthrus {

constexpr int kSampThreads = 1024;
constexpr int kSampTile = 1024;       // elements of one CDF tile
constexpr int kSampMaxTiles = 256;    // vocab <= 262144

__device__ __forceinline__ float warp_incl_scan(float x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = __fadd_rn(x, y);
  }
  return x;
}

// exp((z_k - m) / T): the unnormalised softmax weight at temperature T
struct TemperedWeight {
  const float* z;
  float m, inv_t;
  __device__ __forceinline__ float operator()(int k) const { return expf(__fmul_rn(__fsub_rn(z[k], m), inv_t)); }
};

// max(0, p_k - q_k) with p = softmax(zv / T), q = softmax(zd / T) (row maxima and
// normalisers given)
struct ResidualWeight {
  const float* zv;
  const float* zd;
  float mv, md, inv_t, rzv, rzd;
  __device__ __forceinline__ float operator()(int k) const {
    const float p = __fmul_rn(expf(__fmul_rn(__fsub_rn(zv[k], mv), inv_t)), rzv);
    const float q = __fmul_rn(expf(__fmul_rn(__fsub_rn(zd[k], md), inv_t)), rzd);
    return fmaxf(__fsub_rn(p, q), 0.f);
  }
};

template <class W>
__device__ __forceinline__ void tile_load(const W& w, int s, int V, int lane, float (&x)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int k = s * kSampTile + j * 32 + lane;
    x[j] = k < V ? w(k) : 0.f;
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

// Inverse-CDF draw from the weights w(0..V-1) with the uniform v; the whole CTA
// calls it, the result (or -1 when every weight is zero) is returned to every thread.
template <class W>
__device__ int sample_row(const W& w, int V, float v, SampleSmem& sm) {
  const int nt = (V + kSampTile - 1) / kSampTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int s = warp; s < nt; s += kSampThreads / 32) {
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

// Row maximum of z over a CTA; *bad set if a logit is NaN or +inf.
__device__ float row_max(const float* z, int V, int* bad_s) {
  float m = -INFINITY;
  bool bad = false;
  for (int k = threadIdx.x; k < V; k += kSampThreads) {
    const float x = z[k];
    bad |= !(x < INFINITY);
    m = fmaxf(m, x);
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[kSampThreads / 32];
  if (bad) *bad_s = 1;
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  float r = wm[0];
  for (int i = 1; i < kSampThreads / 32; ++i) r = fmaxf(r, wm[i]);
  __syncthreads();
  return r;
}

// One categorical draw per row: out[r] ~ softmax(logits[r] / T) with uniforms[r].
// A NaN or +inf logit (or a row of -inf only) sets ORTHRUS_ERR_NAN and out[r] = -1.
__global__ void __launch_bounds__(kSampThreads) sample_rows_kernel(const float* logits, int V, float inv_t,
                                                                   const float* uniforms, int* out, int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ SampleSmem sm;
  __shared__ int bad;
  const int row = blockIdx.x;
  const float* z = logits + (size_t)row * V;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const float m = row_max(z, V, &bad);
  if (bad || m == -INFINITY) {
    if (threadIdx.x == 0) {
      out[row] = -1;
      if (status) set_status(status, ORTHRUS_ERR_NAN);
    }
    return;
  }
  const int r = sample_row(TemperedWeight{z, m, inv_t}, V, uniforms[row], sm);
  if (threadIdx.x == 0) out[row] = r;
}

// Row maximum and normaliser Z = sum exp((z - m) / T) of each logits row (online,
// one CTA per row): stats[r] = (m, Z).
__global__ void __launch_bounds__(kSampThreads) row_stats_kernel(const float* dl, int draft_rows, const float* vl,
                                                                 int V, float inv_t, float2* stats, int* status) {
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x;
  const float* z = row < draft_rows ? dl + (size_t)row * V : vl + (size_t)(row - draft_rows) * V;
  float m = -INFINITY, s = 0.f;
  bool bad = false;
  for (int k = threadIdx.x; k < V; k += kSampThreads) {
    const float x = z[k];
    if (!(x < INFINITY)) {
      bad = true;
    } else if (x > m) {
      s = (m == -INFINITY ? 0.f : s * expf((m - x) * inv_t)) + 1.f;
      m = x;
    } else if (x > -INFINITY) {
      s += expf((x - m) * inv_t);
    }
  }
  auto merge = [&](float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
      m = m2;
      s = s2;
    } else if (m2 > m) {
      s = s * expf((m - m2) * inv_t) + s2;
      m = m2;
    } else {
      s += s2 * expf((m2 - m) * inv_t);
    }
  };
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    merge(m2, s2);
  }
  __shared__ float wm[kSampThreads / 32], ws[kSampThreads / 32];
  __shared__ int any_bad;
  if (threadIdx.x == 0) any_bad = 0;
  __syncthreads();
  if (bad) any_bad = 1;
  if ((threadIdx.x & 31) == 0) {
    wm[threadIdx.x >> 5] = m;
    ws[threadIdx.x >> 5] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    m = wm[0];
    s = ws[0];
    for (int i = 1; i < kSampThreads / 32; ++i) merge(wm[i], ws[i]);
    if (any_bad || m == -INFINITY) {
      set_status(status, ORTHRUS_ERR_NAN);
      stats[row] = make_float2(0.f, 1.f);
    } else {
      stats[row] = make_float2(m, s);
    }
  }
}

// Rejection-sampling consensus and commit, one CTA per sequence b. Rows: draft
// logits dl [B][K][V], verify logits vl [B][K+1][V], stats from row_stats_kernel
// (draft rows first). Writes committed [b][0..K] (d_1..d_a, last, then -1),
// accept_len[b] = a, pending[b] = last, len[b] += a + 1. With the status word set
// (by this step or earlier) nothing is committed: accept_len = -1, committed = -1.
__global__ void __launch_bounds__(kSampThreads) accept_sample_kernel(int* pending, const int* draft, const float* dl,
                                                                     const float* vl, const float2* stats, int B,
                                                                     int K, int V, float inv_t, const float* u_acc,
                                                                     const float* u_fin, int* accept_len,
                                                                     int* committed, int* len, int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ SampleSmem sm;
  __shared__ unsigned int masks[2];
  const int b = blockIdx.x, t = threadIdx.x;
  bool acc = false;
  if (t < K) {
    const int d = draft[b * K + t];
    if (d < 0 || d >= V) {
      set_status(status, ORTHRUS_ERR_ARG);
    } else {
      const float2 sd = stats[b * K + t];
      const float2 sv = stats[B * K + b * (K + 1) + t];
      const float eq = expf(__fmul_rn(__fsub_rn(dl[((size_t)b * K + t) * V + d], sd.x), inv_t));
      const float ep = expf(__fmul_rn(__fsub_rn(vl[((size_t)b * (K + 1) + t) * V + d], sv.x), inv_t));
      // u * q < p with q = eq / Zd, p = ep / Zv
      acc = __fmul_rn(__fmul_rn(u_acc[b * K + t], eq), sv.y) < __fmul_rn(ep, sd.y);
    }
  }
  if (t < 64) {
    const unsigned bal = __ballot_sync(0xffffffffu, acc);
    if ((t & 31) == 0) masks[t >> 5] = bal;
  }
  __syncthreads();
  const unsigned long long all = (unsigned long long)masks[0] | ((unsigned long long)masks[1] << 32);
  int a = __ffsll((long long)~all) - 1;  // first rejected draft
  if (a < 0 || a > K) a = K;

  const size_t vrow = (size_t)b * (K + 1) + a;
  const float2 sv = stats[B * K + vrow];
  int last = -1;
  if (a < K) {
    const float2 sd = stats[b * K + a];
    const ResidualWeight w{vl + vrow * V, dl + ((size_t)b * K + a) * V, sv.x, sd.x, inv_t, 1.f / sv.y, 1.f / sd.y};
    last = sample_row(w, V, u_fin[b], sm);
  }
  if (last < 0)  // the bonus row p_K; also p_a if the residual rounded to zero everywhere
    last = sample_row(TemperedWeight{vl + vrow * V, sv.x, inv_t}, V, u_fin[b], sm);

  const bool err = *(volatile const int*)status != 0 || last < 0;
  if (t <= K) {
    int v;
    if (err) v = -1;
    else if (t < a) v = draft[b * K + t];
    else if (t == a) v = last;
    else v = -1;
    committed[b * (K + 1) + t] = v;
  }
  if (t == 0) {
    if (err) {
      accept_len[b] = -1;
    } else {
      accept_len[b] = a;
      pending[b] = last;
      len[b] += a + 1;
    }
  }
}

}  // namespace orthrus
