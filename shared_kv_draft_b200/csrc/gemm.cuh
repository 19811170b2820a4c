// Skinny weight-streaming GEMM on the sm_100a tensor cores:
//     Y[m][n] = sum_k X[m][k] * W[n][k]     (X: tokens x Kd, W: out features x Kd, bf16)
//
// Decode-step GEMMs have few token rows (B*(K+1), e.g. 33) and large weights,
// so they are bound by streaming W from HBM. Design:
//  * "swap AB": 128 weight rows form the MMA's M dimension, tokens its N
//    dimension (Mt = token rows rounded up to 16), so no tensor work is wasted
//    on padding rows of W.
//  * Work = (token tile, weight tile of 128 rows, 64-wide k chunk) units. A
//    persistent grid of one CTA per SM takes an equal contiguous range of units
//    (stream-K), so every SM streams the same number of weight bytes whatever
//    the tile count.
//  * Warp roles: warp 0 issues TMA loads (weight tile 16 KB + token tile per
//    stage, 128-byte swizzle) into a multi-stage mbarrier ring; warp 1 issues
//    tcgen05.mma (one thread) into a double-buffered TMEM accumulator;
//    warps 2-5 drain TMEM (tcgen05.ld) and run the fused epilogue.
//  * A weight tile split between CTAs is finished by whichever contributor
//    arrives last (atomic counter, no waiting): it sums all fp32 partials in a
//    fixed k order, so results do not depend on arrival order.
//  * Epilogues: fp32 store, residual add into the fp32 hidden state, per-head
//    q/k RMSNorm + RoPE + fp16 store of q and of K/V (bf16 values) into the
//    cache (or the draft block scratch), SwiGLU (each tile holds 64 gate rows
//    and the 64 matching up rows; hi and lo planes out), and LM-head argmax
//    (64-bit max of (value, -index)).
//  * X may come in two bf16 planes (hi + lo of one fp32 activation): one MMA
//    per k slice multiplies the weight chunk with both (N = 2 Mt), into two fp32
//    accumulators side by side in TMEM that the epilogue adds.
#pragma once
#include "ptx.cuh"

namespace orthrus {

enum EpiKind : int { EPI_STORE = 0, EPI_RESID = 1, EPI_QKV = 2, EPI_SWIGLU = 3, EPI_ARGMAX = 4 };
enum ViewMode : int { VIEW_DRAFT = 0, VIEW_VERIFY = 1 };

constexpr int kGemmThreads = 192;
constexpr int kEpiStride = 132;  // padded row of the epilogue staging tile (floats)

struct QkvEpi {
  int H, Hkv, d, Q, b0;      // heads, kv heads, head dim, block rows per sequence, first sequence
  int qk_norm, mode;         // mode: VIEW_DRAFT -> K/V into the block scratch rows i; else cache slots len+i
  float eps;
  const float* gq;           // [d]
  const float* gk;           // [d]
  const float2* rope;        // [M][d/2] (cos, sin) of each token row's position
  const int* len;            // [batch] cache lengths
  __half* qbuf;              // [nb][Hkv][Q*G][d], fp16
  __half* kdst;              // this layer's K destination [batch][Hkv][kv_stride][d] (bf16 values, fp16 encoding)
  __half* vdst;
  int kv_stride;             // capacity (cache) or block-scratch rows
};

struct GemmArgs {
  int N, Kd, M;              // weight rows, reduction length, valid token rows
  int Mt, mt_alloc;          // token tile (multiple of 16, <= 128), TMEM columns per accumulator (>= planes Mt)
  int m_tiles, n_tiles, k_chunks;
  long long total_units;
  int stages;
  int planes;                // activation planes of X: 2 (hi + lo rows in one MMA of N = 2 Mt) or 1
  int swiglu_F;              // SwiGLU: row offset of the up rows in W
  float* partial;            // [2 * grid][128 rows][Mt] fp32 partial sums of split tiles
  int* tile_counter;         // [m_tiles * n_tiles], zero between launches
  int* status;
  float* out_f32;            // STORE: Y[M][ld_out]; RESID: h[M][ld_out] (+=)
  int ld_out;
  __nv_bfloat16* out_bf16;   // SWIGLU: act[2][M][ld_out], hi plane then the lo plane at + out_lo
  size_t out_lo;
  QkvEpi qkv;
  unsigned long long* amax;  // ARGMAX: [M] running keys
  float* logits;             // ARGMAX: optional fp32 [M][ld_logits]
  long long ld_logits;
};

__host__ __device__ inline long long unit_start(long long W, int G, int c) { return (W * c) / G; }

// CTA that owns unit u under the equal contiguous split of W units over G CTAs.
__device__ inline int unit_owner(long long u, long long W, int G) {
  int c = (int)((u * G) / W);
  while (c + 1 < G && unit_start(W, G, c + 1) <= u) ++c;
  while (c > 0 && unit_start(W, G, c) > u) --c;
  return c;
}

__host__ inline size_t gemm_smem_bytes(int Mt, int stages, int planes) {
  return 1024 /*align*/ + (size_t)stages * (16384 + (size_t)Mt * 128 * planes) + 32 * kEpiStride * 4 + 4 * 32 * 8 +
         2 * 16 * 8 + 128;
}

// --------------------------------------------------------------------------
// epilogue on 32 token columns [m0, m0+32) of one 128-row tile; thread `row`
// holds v[j] = Y[tile token m0 + j][tile row `row`]
// --------------------------------------------------------------------------
template <int EPI>
__device__ __forceinline__ void epilogue_group(const GemmArgs& a, float* v, int row, int m0, int mt, int nt,
                                               int m_valid, float* epi, unsigned long long* red) {
  const int ew = (threadIdx.x >> 5) - 2;  // epilogue warp 0..3
  const int lane = threadIdx.x & 31;
  if constexpr (EPI == EPI_STORE || EPI == EPI_RESID) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int m = m0 + j;
      if (m < m_valid) {
        float* p = a.out_f32 + (size_t)(mt * 128 + m) * a.ld_out + nt * 128 + row;
        if constexpr (EPI == EPI_STORE) *p = v[j];
        else *p += v[j];
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // rows 0..63 = gate rows nt*64.., rows 64..127 = the matching up rows
    if (row >= 64) {
#pragma unroll
      for (int j = 0; j < 32; ++j) epi[j * kEpiStride + (row - 64)] = v[j];
    }
    named_bar_sync(1, 128);
    if (row < 64) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int m = m0 + j;
        if (m < m_valid) {
          const float g = v[j];
          const float u = epi[j * kEpiStride + row];
          const float s = g / (1.0f + __expf(-g));
          const float y = s * u;
          const __nv_bfloat16 yh = __float2bfloat16(y);
          const size_t o = (size_t)(mt * 128 + m) * a.ld_out + nt * 64 + row;
          a.out_bf16[o] = yh;
          a.out_bf16[a.out_lo + o] = __float2bfloat16(y - __bfloat162float(yh));
        }
      }
    }
    named_bar_sync(1, 128);
  } else if constexpr (EPI == EPI_QKV) {
    const QkvEpi& q = a.qkv;
#pragma unroll
    for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j];
    named_bar_sync(1, 128);
    const int d = q.d;
    const int nper = d >> 5;  // values per lane: 2 (d=64) or 4 (d=128)
    const int half = d >> 1;
    const int G = q.H / q.Hkv;
    for (int j = ew; j < 32; j += 4) {
      const int m = m0 + j;
      if (m >= m_valid) break;
      const int grow = mt * 128 + m;  // token row in the block
      const int bb = grow / q.Q, i = grow - bb * q.Q;
      const int b = q.b0 + bb;
      for (int hl = 0; hl < 128 / d; ++hl) {
        const int hh = (nt * 128) / d + hl;  // head index in the fused q|k|v rows
        const int kind = hh < q.H ? 0 : (hh < q.H + q.Hkv ? 1 : 2);
        float x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < nper) x[k] = epi[j * kEpiStride + hl * d + lane + 32 * k];
        if (kind < 2) {
          if (q.qk_norm) {
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (k < nper) ss += x[k] * x[k];
            ss = warp_sum(ss);
            const float r = rsqrtf(ss / (float)d + q.eps);
            const float* g = kind == 0 ? q.gq : q.gk;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (k < nper) x[k] = x[k] * r * g[lane + 32 * k];
          }
          // rotate-half RoPE: element e pairs with e + d/2 (same lane, k and k + nper/2)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (k < nper / 2) {
              const int e = lane + 32 * k;
              const float2 cs = q.rope[(size_t)grow * half + e];
              const float x1 = x[k], x2 = x[k + nper / 2];
              x[k] = x1 * cs.x - x2 * cs.y;
              x[k + nper / 2] = x2 * cs.x + x1 * cs.y;
            }
          }
        }
        if (kind == 0) {
          const int kvh = hh / G, g = hh - kvh * G;
          __half* dst = q.qbuf + ((size_t)(bb * q.Hkv + kvh) * (q.Q * G) + i * G + g) * d;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < nper) dst[lane + 32 * k] = __float2half_rn(x[k]);
        } else {
          const int kvh = hh - q.H - (kind == 2 ? q.Hkv : 0);
          const int slot = q.mode == VIEW_DRAFT ? i : q.len[b] + i;
          if (slot >= 0 && slot < q.kv_stride) {
            __half* base = kind == 1 ? q.kdst : q.vdst;
            __half* dst = base + ((size_t)(b * q.Hkv + kvh) * q.kv_stride + slot) * d;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (k < nper) dst[lane + 32 * k] = __float2half_rn(kv_value(x[k]));
          }
        }
      }
    }
    named_bar_sync(1, 128);
  } else if constexpr (EPI == EPI_ARGMAX) {
    const uint32_t col = nt * 128 + row;  // vocabulary index
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int m = m0 + j;
      unsigned long long key = 0ull;
      if (m < m_valid) {
        if (a.logits) a.logits[(size_t)(mt * 128 + m) * a.ld_logits + col] = v[j];
        if (isnan(v[j])) set_status(a.status, ORTHRUS_ERR_NAN);
        else key = argmax_key(v[j], col);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) key = ull_max(key, __shfl_xor_sync(0xffffffffu, key, o));
      if (lane == 0) red[ew * 32 + j] = key;
    }
    named_bar_sync(1, 128);
    if (ew == 0) {
      const int m = m0 + lane;
      unsigned long long k = ull_max(ull_max(red[lane], red[32 + lane]), ull_max(red[64 + lane], red[96 + lane]));
      if (m < m_valid && k != 0ull) atomicMax(a.amax + mt * 128 + m, k);
    }
    named_bar_sync(1, 128);
  }
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int S = a.stages;
  const uint32_t x_bytes = (uint32_t)a.Mt * 128u * (uint32_t)a.planes;  // [plane][Mt rows][64]
  const uint32_t stage_bytes = 16384u + x_bytes;
  float* epi = (float*)(smem + (size_t)S * stage_bytes);
  unsigned long long* red = (unsigned long long*)(epi + 32 * kEpiStride);
  uint64_t* full = (uint64_t*)(red + 128);
  uint64_t* empty = full + 16;
  uint64_t* accf = empty + 16;  // [2]
  uint64_t* acce = accf + 2;    // [2]
  uint64_t* done = acce + 2;
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  int* flag = (int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const long long W = a.total_units;
  const long long u0 = unit_start(W, G, c), u1 = unit_start(W, G, c + 1);
  const int kc = a.k_chunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * a.mt_alloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int issued[16];
      for (int s = 0; s < 16; ++s) issued[s] = -1;
      auto load_w = [&](int s, long long u) {
        const int t = (int)(u / kc), k = (int)(u - (long long)t * kc);
        const int nt = t / a.m_tiles;
        uint8_t* wdst = smem + (size_t)s * stage_bytes;
        if constexpr (EPI == EPI_SWIGLU) {
          tma_load_2d_hint(wdst, &tmW, &full[s], k * 64, nt * 64, pol_w);
          tma_load_2d_hint(wdst + 8192, &tmW, &full[s], k * 64, a.swiglu_F + nt * 64, pol_w);
        } else {
          tma_load_2d_hint(wdst, &tmW, &full[s], k * 64, nt * 128, pol_w);
        }
      };
      auto load_x = [&](int s, long long u) {
        const int t = (int)(u / kc), k = (int)(u - (long long)t * kc);
        const int mt = t - (t / a.m_tiles) * a.m_tiles;
        uint8_t* xdst = smem + (size_t)s * stage_bytes + 16384;
        if (a.planes == 2) tma_load_3d(xdst, &tmX, &full[s], k * 64, mt * 128, 0);  // Mt rows of both planes
        else tma_load_2d_hint(xdst, &tmX, &full[s], k * 64, mt * 128, pol_x);  // one box of Mt token rows
      };
      // weights never depend on earlier kernels: fill the ring with weight tiles
      // before waiting for the predecessor, then add the activation tiles
      const int pre = (int)min((long long)S, u1 - u0);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], stage_bytes);
        load_w(i, u0 + i);
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i) {
        load_x(i, u0 + i);
        issued[i] = 0;
      }
      int it = pre;
      for (long long u = u0 + pre; u < u1; ++u, ++it) {
        const int s = it % S, ph = (it / S) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        load_w(s, u);
        load_x(s, u);
        issued[s] = ph;
      }
      // every load issued must have landed before the CTA may exit
      for (int s = 0; s < S && s < 16; ++s)
        if (issued[s] >= 0) mbar_wait(&full[s], (uint32_t)issued[s], a.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // with two planes the B operand is the Mt hi rows then the Mt lo rows: one MMA of N = 2 Mt
      const uint32_t idesc = idesc_bf16(128, a.planes * a.Mt, false);
      int it = 0, seg = 0;
      long long u = u0;
      bool ok = true;
      while (ok && u < u1) {
        const int t = (int)(u / kc);
        const long long seg_start = u, seg_end = min(u1, (long long)(t + 1) * kc);
        const int buf = seg & 1, use = seg >> 1;
        if (!mbar_wait(&acce[buf], (use & 1) ^ 1, a.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * a.mt_alloc;
        for (; u < seg_end; ++u, ++it) {
          const int s = it % S, ph = (it / S) & 1;
          if (!mbar_wait(&full[s], ph, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(smem + (size_t)s * stage_bytes);
          const uint32_t xa = wa + 16384;
          // 32-byte k steps: (32 >> 4) added to the descriptors' start-address field
          const uint64_t wd0 = sw128_desc(wa, 16, 1024), xd0 = sw128_desc(xa, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(d_tmem, wd0 + (uint64_t)(2 * kk), xd0 + (uint64_t)(2 * kk), idesc, (u > seg_start || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&accf[buf]);
        ++seg;
      }
      mma_commit(done);
      mbar_wait(done, 0, a.status);
    }
  } else {
    // ---------------- epilogue warps ----------------
    griddep_wait();  // outputs and shared scratch are touched only after the predecessor finished
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    // accumulator columns [col, col + 32); with two planes the lo products sit Mt columns on
    auto acc_ld = [&](uint32_t taddr, int col, float* v) {
      tmem_ld32(taddr + col, v);
      if (a.planes == 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float w[16];
          tmem_ld16(taddr + a.Mt + col + 16 * h, w);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[16 * h + j] += w[j];
        }
      }
    };
    int seg = 0;
    long long u = u0;
    const int first_tile = (int)(u0 / kc);
    while (u < u1) {
      const int t = (int)(u / kc);
      const long long seg_start = u, seg_end = min(u1, (long long)(t + 1) * kc);
      u = seg_end;
      const int buf = seg & 1, use = seg >> 1;
      ++seg;
      // one thread waits so that all four warps take the same branch (a named
      // barrier with a missing warp would never complete)
      if (threadIdx.x == 64) flag[1 + buf] = mbar_wait(&accf[buf], use & 1, a.status) ? 1 : 0;
      named_bar_sync(1, 128);
      const bool got = flag[1 + buf] != 0;
      tc_fence_after();
      const int nt = t / a.m_tiles, mt = t - nt * a.m_tiles;
      const int m_valid = min(a.Mt, a.M - mt * 128);
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * a.mt_alloc;
      const bool whole = seg_start == (long long)t * kc && seg_end == (long long)(t + 1) * kc;
      float v[32];
      if (!got) break;
      if (whole) {
        for (int m0 = 0; m0 < a.Mt; m0 += 32) {
          acc_ld(taddr, m0, v);
          epilogue_group<EPI>(a, v, row, m0, mt, nt, m_valid, epi, red);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[buf]);
      } else {
        // write this CTA's partial sum of the tile, then count arrivals
        // this thread's Mt partial sums, contiguous: [slot][row][Mt]
        const int slot = 2 * c + (t == first_tile ? 0 : 1);
        float* part = a.partial + (size_t)slot * (128 * 128) + (size_t)row * a.Mt;
        for (int m0 = 0; m0 < a.Mt; m0 += 32) {
          acc_ld(taddr, m0, v);
          const int n4 = min(32, a.Mt - m0) / 4;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < n4) __stcg(reinterpret_cast<float4*>(part + m0) + q, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[buf]);
        const int c_lo = unit_owner((long long)t * kc, W, G);
        const int c_hi = unit_owner((long long)(t + 1) * kc - 1, W, G);
        __threadfence();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          const int old = atomicAdd(a.tile_counter + t, 1);
          *flag = (old == c_hi - c_lo) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (*flag) {
          __threadfence();
          if (threadIdx.x == 64) a.tile_counter[t] = 0;
          for (int m0 = 0; m0 < a.Mt; m0 += 32) {
            const int n4 = min(32, a.Mt - m0) / 4;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
            for (int cc = c_lo; cc <= c_hi; ++cc) {  // fixed k order: the sum does not depend on arrival order
              const int ft = (int)(unit_start(W, G, cc) / kc);
              const float4* pp = reinterpret_cast<const float4*>(
                  a.partial + (size_t)(2 * cc + (t == ft ? 0 : 1)) * (128 * 128) + (size_t)row * a.Mt + m0);
              float4 x[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) x[q] = q < n4 ? __ldcg(pp + q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                v[4 * q] += x[q].x;
                v[4 * q + 1] += x[q].y;
                v[4 * q + 2] += x[q].z;
                v[4 * q + 3] += x[q].w;
              }
            }
            epilogue_group<EPI>(a, v, row, m0, mt, nt, m_valid, epi, red);
          }
        }
        named_bar_sync(1, 128);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * a.mt_alloc);
  }
}

}  // namespace orthrus
