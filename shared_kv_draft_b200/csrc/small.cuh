// Small kernels of the decode step: block embedding (+ RoPE table and the
// capacity check), RMSNorm to bf16 hi/lo planes, argmax finalisation, greedy
// consensus with the KV commit, and dead-slot poisoning.
#pragma once
#include "ptx.cuh"

namespace orthrus {

enum BlockKind : int { BLOCK_DRAFT = 0, BLOCK_VERIFY = 1, BLOCK_PREFILL = 2 };

struct EmbedArgs {
  int kind, nb, b0, Q, D, d, V, mask_id, cap;
  double theta;
  const int* pending;   // [batch]            (draft, verify)
  const int* draft;     // verify: [nb][Q-1]; draft: nullable [nb][Q], previous drafts
  const int* tokens;    // prefill: tokens[b * tok_stride + tok_off + i]
  int tok_stride, tok_off;
  const int* len;       // [batch]
  const __nv_bfloat16* embed;
  float* h;             // [M][D]
  float2* rope;         // [M][d/2]
  int* status;
};

// Block row m = bb*Q + i holds sequence b0+bb at position len[b]+i:
//   draft:   ids [y, MASK x (Q-1)], or [y, d_1 .. d_{Q-1}] of the previous drafts
//            (draft [nb][Q]) in a refinement step
//   verify:  ids [y, d_1 .. d_{Q-1}]
//   prefill: prompt tokens
__global__ void embed_kernel(const EmbedArgs a) {
  griddep_wait();
  griddep_launch();
  const int m = blockIdx.x;
  const int bb = m / a.Q, i = m - bb * a.Q;
  const int b = a.b0 + bb;
  int id;
  if (a.kind == BLOCK_PREFILL) id = a.tokens[(size_t)b * a.tok_stride + a.tok_off + i];
  else if (i == 0) id = a.pending[b];
  else if (a.kind != BLOCK_DRAFT) id = a.draft[bb * (a.Q - 1) + (i - 1)];
  else id = a.draft ? a.draft[bb * a.Q + (i - 1)] : a.mask_id;  // refinement: previous drafts
  if (id < 0 || id >= a.V) {
    if (threadIdx.x == 0) set_status(a.status, ORTHRUS_ERR_ARG);
    id = 0;
  }
  const int n = a.len[b];
  if (threadIdx.x == 0 && i == 0 && a.kind != BLOCK_DRAFT && n + a.Q > a.cap) set_status(a.status, ORTHRUS_ERR_CAPACITY);
  const __nv_bfloat16* src = a.embed + (size_t)id * a.D;
  float* dst = a.h + (size_t)m * a.D;
  for (int c = threadIdx.x * 8; c < a.D; c += blockDim.x * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(src + c);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float4 lo, hi;
    float2 f0 = __bfloat1622float2(p[0]), f1 = __bfloat1622float2(p[1]);
    float2 f2 = __bfloat1622float2(p[2]), f3 = __bfloat1622float2(p[3]);
    lo = make_float4(f0.x, f0.y, f1.x, f1.y);
    hi = make_float4(f2.x, f2.y, f3.x, f3.y);
    *reinterpret_cast<float4*>(dst + c) = lo;
    *reinterpret_cast<float4*>(dst + c + 4) = hi;
  }
  // RoPE angles pos * theta^(-2j/d), evaluated in double and rounded to fp32
  const int half = a.d / 2;
  const double pos = (double)(n + i);
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const double ang = pos * pow(a.theta, -2.0 * (double)j / (double)a.d);
    a.rope[(size_t)m * half + j] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// x = h[src_first + m*src_stride] * rsqrt(mean(h^2) + eps) * gain -> out[m] = bf16(x), and with
// out_lo > 0 also the lo plane out[out_lo + m] = bf16(x - bf16(x)); optionally zero keys[m]
__global__ void rmsnorm_kernel(const float* __restrict__ h, int D, const float* __restrict__ gain, float eps,
                               __nv_bfloat16* __restrict__ out, size_t out_lo, int src_first, int src_stride,
                               unsigned long long* reset_keys) {
  griddep_wait();
  griddep_launch();
  const int m = blockIdx.x;
  const float* x = h + (size_t)(src_first + m * src_stride) * D;
  __shared__ float red[32];
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float r = rsqrtf(red[0] / (float)D + eps);
  __nv_bfloat16* y = out + (size_t)m * D;
  for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + c);
    const float4 g = *reinterpret_cast<const float4*>(gain + c);
    uint32_t h0, h1, l0, l1;
    split_bf16x2(v.x * r * g.x, v.y * r * g.y, h0, l0);
    split_bf16x2(v.z * r * g.z, v.w * r * g.w, h1, l1);
    *reinterpret_cast<uint2*>(y + c) = make_uint2(h0, h1);
    if (out_lo) *reinterpret_cast<uint2*>(y + out_lo + c) = make_uint2(l0, l1);
  }
  if (reset_keys && threadIdx.x == 0) reset_keys[m] = 0ull;
}

// token id = lowest index of the row maximum, from the packed 64-bit keys
__global__ void argmax_finalize_kernel(const unsigned long long* keys, int M, int* dst, int* status) {
  griddep_wait();
  griddep_launch();
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= M) return;
  const unsigned long long k = keys[m];
  if (k == 0ull) {
    set_status(status, ORTHRUS_ERR_NAN);
    dst[m] = 0;
  } else {
    dst[m] = (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
  }
}

// Greedy consensus for sequence b (one CTA of 96 threads, K <= 64):
//   a = number of leading i with d_{i+1} == g_i; commit d_1..d_a, g_a;
//   len += a + 1; pending = g_a. Nothing is committed once the status word
//   holds an error (the verify block may not have been written).
__global__ void accept_kernel(int* pending, const int* draft, const int* ar, int K, int* accept_len, int* committed,
                              int* len, const int* status) {
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x, t = threadIdx.x;
  __shared__ unsigned int masks[3];
  const bool match = t < K && draft[b * K + t] == ar[b * (K + 1) + t];
  const unsigned int bal = __ballot_sync(0xffffffffu, match);
  if ((t & 31) == 0) masks[t >> 5] = bal;
  __syncthreads();
  const unsigned long long all = (unsigned long long)masks[0] | ((unsigned long long)masks[1] << 32);
  int a = __ffsll((long long)~all) - 1;  // index of the first mismatch
  if (a < 0 || a > K) a = K;
  const bool err = *(volatile const int*)status != 0;
  if (t <= K) {
    int v;
    if (err) v = -1;
    else if (t < a) v = draft[b * K + t];
    else if (t == a) v = ar[b * (K + 1) + a];
    else v = -1;
    committed[b * (K + 1) + t] = v;
  }
  if (t == 0) {
    if (err) {
      accept_len[b] = -1;
    } else {
      accept_len[b] = a;
      pending[b] = ar[b * (K + 1) + a];
      len[b] += a + 1;
    }
  }
}

// Overwrite the dead verify slots [len, len + K - a) of every layer and KV head
// with NaN (fp16 0x7E00), after accept_kernel advanced len.
__global__ void poison_kernel(__half* kc, __half* vc, const int* len, const int* accept_len, int K,
                              int B, int Hkv, int cap, int d) {
  griddep_wait();
  griddep_launch();
  const int z = blockIdx.x;  // (l * B + b) * Hkv + h
  const int b = (z / Hkv) % B;
  const int a = accept_len[b];
  if (a < 0) return;
  const int lo = len[b], hi = min(cap, len[b] + K - a);
  const __half nan = __ushort_as_half((unsigned short)0x7E00);
  for (int s = lo; s < hi; ++s) {
    for (int e = threadIdx.x; e < d; e += blockDim.x) {
      kc[((size_t)z * cap + s) * d + e] = nan;
      vc[((size_t)z * cap + s) * d + e] = nan;
    }
  }
}

__global__ void set_len_kernel(int* len, int b, int value) {
  griddep_wait();
  griddep_launch();
  len[b] = value;
}

}  // namespace orthrus
