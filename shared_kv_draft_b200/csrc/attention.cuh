// GQA block attention for the Orthrus decode step on sm_100a.
//
// For one sequence b and KV head kvh, the G query heads x Q block positions
// form the rows of one MMA tile: row r = i*G + g (block position i, query head
// kvh*G + g). Up to 128 rows per tile, so at K = 32 the draft block (32 x 4
// heads) is exactly one tcgen05 M=128 tile.
//   draft view : every row sees cache[0, len) and all Q rows of the block's own
//                draft-view K/V (bidirectional inside the block; Orthrus's
//                diffusion view attends to the shared cache plus the block).
//   verify view: the block's base K/V already sit in cache slots [len, len+Q);
//                row i sees cache[0, len+i] (causal).
// Keys are split into chunks at absolute positions (fixed chunk size per
// launch); each CTA runs one (b, kvh, row tile, chunk):
//   warp 0: TMA loads of the Q tile and of 128-key K/V tiles (double buffer);
//   warp 1: one thread issues S = Q K^T (tcgen05, K-major operands) into TMEM
//           and then O_t = P V (V as an MN-major operand) into TMEM;
//   warps 2-5: one thread per row: online softmax on S read from TMEM, P written
//           as fp16 into shared memory in the 128-byte-swizzled K-major layout,
//           O accumulated in registers with the running rescale.
// Operands are fp16 (q, P, and K/V, whose bf16 values are held in the fp16
// encoding); the output is written as two bf16 planes (hi, lo) for the O projection.
// Chunks are combined by the last CTA to finish (atomic counter, fixed order).
// Cache rows past the visible range inside a loaded tile (stale, NaN-poisoned or
// never written) are masked out of S and their V rows zeroed before P V, so they
// cannot reach the output.
#pragma once
#include "ptx.cuh"

namespace orthrus {

constexpr int kAttnThreads = 192;

struct AttnArgs {
  int B, Hkv, G, Q, d, mode;   // mode: VIEW_DRAFT (0) / VIEW_VERIFY (1)
  int b0;                      // first sequence (index into len and the cache's batch)
  int rows, row_tiles;         // Q*G, ceil(rows / 128)
  int chunk_keys;              // keys per chunk (multiple of 128)
  int cap;                     // cache capacity (keys)
  int z_cache;                 // z coordinate of (b = 0, kvh = 0) in the cache maps: layer * batch * Hkv
  int z_blk;                   // same for the block-scratch maps
  int max_chunks;              // gridDim.x
  float scale_log2;            // log2(e) / sqrt(d)
  const int* len;
  __nv_bfloat16* out;          // [2][nb*Q][H*d]: hi plane, then the lo plane at + out_lo
  size_t out_lo;
  float* part_o;               // [nb*Hkv*row_tiles][max_chunks][128][d]
  float2* part_ml;             // [nb*Hkv*row_tiles][max_chunks][128]
  int* counter;                // [nb*Hkv*row_tiles], zero between launches
  int* status;
};

__host__ inline size_t attn_smem_bytes(int d) {
  // Q tile + 2 stages x (K tile + V tile) + P tile + barriers
  return 1024 + (size_t)128 * d * 2 + 2 * 2 * (size_t)128 * d * 2 + 128 * 128 * 2 + 256;
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                     const __grid_constant__ CUtensorMap tmVb, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int d = D;
  const uint32_t tile_bytes = 128u * d * 2u;  // 128 rows x d fp16
  uint8_t* sQ = smem;
  uint8_t* sK[2] = {smem + tile_bytes, smem + 3 * tile_bytes};
  uint8_t* sV[2] = {smem + 2 * tile_bytes, smem + 4 * tile_bytes};
  uint8_t* sP = smem + 5 * tile_bytes;  // 128 rows x 128 keys fp16 = 32 KB
  uint64_t* bars = (uint64_t*)(sP + 128 * 128 * 2);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* o_full = bars + 7;
  uint64_t* t_done = bars + 8;
  uint64_t* done = bars + 9;
  uint32_t* tmem_slot = (uint32_t*)(bars + 10);
  int* flag = (int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, rt = blockIdx.y;
  const int bh = blockIdx.z;  // local sequence * Hkv + kvh
  const int bb = bh / a.Hkv, kvh = bh - bb * a.Hkv;
  const int b = a.b0 + bb;
  griddep_wait();  // q, the cache and len come from earlier kernels
  griddep_launch();
  const int n = a.len[b];

  // ---- key range of this CTA ------------------------------------------------
  const int row_lo = rt * 128;
  const int row_hi = min(a.rows, row_lo + 128);  // exclusive
  const int i_max = (row_hi - 1) / a.G;           // last block position in this row tile
  int n_chunks, key_lo, key_hi;                   // [key_lo, key_hi) within the source
  bool blk = false;
  if (a.mode == 1) {
    const int kv_end = min(n + i_max + 1, a.cap);
    n_chunks = max(1, (kv_end + a.chunk_keys - 1) / a.chunk_keys);
    key_lo = chunk * a.chunk_keys;
    key_hi = min(kv_end, key_lo + a.chunk_keys);
  } else {
    const int nc = (min(n, a.cap) + a.chunk_keys - 1) / a.chunk_keys;
    n_chunks = nc + 1;
    if (chunk < nc) {
      key_lo = chunk * a.chunk_keys;
      key_hi = min(min(n, a.cap), key_lo + a.chunk_keys);
    } else {
      blk = true;
      key_lo = 0;
      key_hi = a.Q;
    }
  }
  if (chunk >= n_chunks) return;  // uniform across the CTA, before any barrier or TMEM use
  const int n_tiles = (key_hi - key_lo + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    mbar_init(t_done, 4);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base;        // S: 128 columns
  const uint32_t tO = tmem_base + 128;  // O tile: d columns

  const int zc = a.z_cache + b * a.Hkv + kvh;
  const int zb = a.z_blk + b * a.Hkv + kvh;
  constexpr int halves = d / 64;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      mbar_arrive_expect_tx(q_full, tile_bytes);
      const int qrow = bh * a.rows + row_lo;
      for (int h = 0; h < halves; ++h) tma_load_2d(sQ + h * 16384, &tmQ, q_full, h * 64, qrow);
      int issued[2] = {-1, -1};
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1, ph = (j >> 1) & 1;
        if (!mbar_wait(&kv_empty[s], ph ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * tile_bytes);
        const int key0 = key_lo + j * 128;
        for (int h = 0; h < halves; ++h) {
          if (blk) {
            tma_load_3d(sK[s] + h * 16384, &tmKb, &kv_full[s], h * 64, key0, zb);
            tma_load_3d(sV[s] + h * 16384, &tmVb, &kv_full[s], h * 64, key0, zb);
          } else {
            tma_load_3d(sK[s] + h * 16384, &tmK, &kv_full[s], h * 64, key0, zc);
            tma_load_3d(sV[s] + h * 16384, &tmV, &kv_full[s], h * 64, key0, zc);
          }
        }
        issued[s] = ph;
      }
      mbar_wait(q_full, 0, a.status);
      for (int s = 0; s < 2; ++s)
        if (issued[s] >= 0) mbar_wait(&kv_full[s], (uint32_t)issued[s], a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idS = idesc_f16(128, 128, false);  // fp16 q and K
      const uint32_t idO = idesc_f16(128, d, true);      // fp16 P and V
      bool ok = mbar_wait(q_full, 0, a.status);
      const uint32_t qa = smem_u32(sQ), pa = smem_u32(sP);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1, ph = (j >> 1) & 1;
        if (!mbar_wait(&kv_full[s], ph, a.status)) break;
        if (j > 0 && !mbar_wait(t_done, (j - 1) & 1, a.status)) break;  // S, O tile and P free again
        tc_fence_after();
        const uint32_t ka = smem_u32(sK[s]), va = smem_u32(sV[s]);
        for (int kk = 0; kk < d / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tS, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        if (!mbar_wait(p_full, j & 1, a.status)) break;
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per MMA
          const uint32_t poff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tO, sw128_desc(pa + poff, 16, 1024), sw128_desc(va + kk * 2048, 16384, 1024), idO,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(o_full);
        mma_commit(&kv_empty[s]);
      }
      mma_commit(done);
      mbar_wait(done, 0, a.status);
    }
  } else {
    // ---- softmax / accumulation warps: thread = query row --------------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // row within the tile (TMEM lane)
    const int grow = row_lo + r;         // row within (b, kvh)
    const bool row_ok = grow < a.rows;
    const int i = row_ok ? grow / a.G : 0;
    // number of visible keys of this row within the source
    int lim;
    if (a.mode == 1) lim = min(n + i + 1, key_hi);
    else lim = key_hi;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float o[d];
#pragma unroll
    for (int e = 0; e < d; ++e) o[e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (threadIdx.x == 64) flag[j & 1] = mbar_wait(s_full, j & 1, a.status) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!flag[j & 1]) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = key_lo + j * 128;
      const int s = j & 1;
      // pass 1: row max of the visible scores
      float mx = -INFINITY;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float v[32];
        tmem_ld32(tS + lane_base + c0, v);
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (key0 + c0 + t < lim) mx = fmaxf(mx, v[t] * a.scale_log2);
      }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
      // pass 2: P = exp2(s - m_new) as fp16 into the swizzled P tile
      float sum = 0.f;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float v[32];
        tmem_ld32(tS + lane_base + c0, v);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const float p0 = (key0 + c0 + t < lim) ? exp2f(v[t] * a.scale_log2 - m_new) : 0.f;
          const float p1 = (key0 + c0 + t + 1 < lim) ? exp2f(v[t + 1] * a.scale_log2 - m_new) : 0.f;
          sum += p0 + p1;
          __half2 h2 = __floats2half2_rn(p0, p1);
          pk[t / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        // keys c0..c0+31 = four 16-byte chunks of row r in atom column c0/64
        const int ac = c0 >> 6;
        uint8_t* rowp = sP + ac * 16384 + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk16 = ((c0 & 63) >> 3) + q4;
          uint4 val = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          *reinterpret_cast<uint4*>(rowp + ((chunk16 ^ (r & 7)) << 4)) = val;
        }
      }
      l_run = l_run * alpha + sum;
      // V rows of keys nobody may see are zeroed (thread r owns key row r of the tile)
      {
        const int key_valid_end = (a.mode == 1) ? min(n + i_max + 1, key_hi) : key_hi;
        if (key0 + r >= key_valid_end) {
          for (int h = 0; h < halves; ++h) {
            uint4* vr = reinterpret_cast<uint4*>(sV[s] + h * 16384 + r * 128);
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) vr[q8] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (threadIdx.x == 64) flag[2 + (j & 1)] = mbar_wait(o_full, j & 1, a.status) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!flag[2 + (j & 1)]) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < d; c0 += 32) {
        float v[32];
        tmem_ld32(tO + lane_base + c0, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) o[c0 + t] = o[c0 + t] * alpha + v[t];
      }
      m_run = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_done);
    }

    if (ok) {
      const int H = a.Hkv * a.G;
      const int g = grow - i * a.G;
      __nv_bfloat16* dst = a.out + ((size_t)(bb * a.Q + i) * H + kvh * a.G + g) * d;
      if (n_chunks == 1) {
        if (row_ok) {
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
          for (int e = 0; e < d; e += 8) {
            float y8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) y8[t] = o[e + t] * inv;
            st_split_x8(dst + e, dst + a.out_lo + e, y8);
          }
        }
      } else {
        const int slot = bh * a.row_tiles + rt;
        // partial O as [chunk][d/4][128 rows][4]: a warp's float4 stores (and the merge's
        // loads) are 512 contiguous bytes
        float4* po = reinterpret_cast<float4*>(a.part_o) + ((size_t)slot * a.max_chunks + chunk) * (d / 4) * 128 + r;
#pragma unroll
        for (int e = 0; e < d; e += 4) po[(size_t)(e / 4) * 128] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        a.part_ml[((size_t)slot * a.max_chunks + chunk) * 128 + r] = make_float2(m_run, l_run);
        __threadfence();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          const int old = atomicAdd(a.counter + slot, 1);
          flag[4] = (old == n_chunks - 1) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (flag[4]) {
          __threadfence();
          if (threadIdx.x == 64) a.counter[slot] = 0;
          if (row_ok) {
            // chunks merged in chunk order; the weights first, then O in 64-column halves
            // with two chunks' loads in flight
            const float2* ml_row = a.part_ml + (size_t)slot * a.max_chunks * 128 + r;
            float mstar = -INFINITY;
            for (int cc = 0; cc < n_chunks; ++cc) mstar = fmaxf(mstar, __ldcg(ml_row + (size_t)cc * 128).x);
            float L = 0.f;
            for (int cc = 0; cc < n_chunks; ++cc) {
              const float2 ml = __ldcg(ml_row + (size_t)cc * 128);
              L += ml.y * ((ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mstar));
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            const float4* p4 = reinterpret_cast<const float4*>(a.part_o) + (size_t)slot * a.max_chunks * (d / 4) * 128 + r;
#pragma unroll 1
            for (int h = 0; h < d / 64; ++h) {
              float acc[64];
#pragma unroll
              for (int e = 0; e < 64; ++e) acc[e] = 0.f;
#pragma unroll 2
              for (int cc = 0; cc < n_chunks; ++cc) {
                const float2 ml = __ldcg(ml_row + (size_t)cc * 128);
                const float w = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mstar);
                const float4* pc = p4 + ((size_t)cc * (d / 4) + h * 16) * 128;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const float4 x = __ldcg(pc + (size_t)e * 128);
                  acc[4 * e] += x.x * w;
                  acc[4 * e + 1] += x.y * w;
                  acc[4 * e + 2] += x.z * w;
                  acc[4 * e + 3] += x.w * w;
                }
              }
#pragma unroll
              for (int e = 0; e < 64; e += 8) {
                float y8[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) y8[t] = acc[e + t] * inv;
                st_split_x8(dst + h * 64 + e, dst + a.out_lo + h * 64 + e, y8);
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace orthrus
