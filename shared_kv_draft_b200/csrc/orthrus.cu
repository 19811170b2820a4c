// Host side of liborthrus: plan construction (TMA descriptors encoded once),
// launch geometry, the forward orchestration of the draft / verify / prefill
// passes, and the C-ABI entry points declared in include/orthrus.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <utility>
#include <vector>

#include "attention.cuh"
#include "forward.cuh"
#include "gemm.cuh"
#include "orthrus.h"
#include "sampling.cuh"
#include "small.cuh"
#include "policy.cuh"

using namespace orthrus;

namespace {

// ---------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link against libcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapDataType kF16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;

// 2D map of 16-bit elements over a row-major [rows][cols] matrix; box = box_cols x box_rows,
// 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
           CUtensorMapDataType dt = kBF16) {
  EncodeTiledFn f = encode_fn();
  if (!f || !base) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return f(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map of 16-bit elements over [z][rows][cols]; box = 64 cols x box_rows rows x box_z.
bool map3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t z, uint32_t box_rows = 128,
           uint32_t box_z = 1, CUtensorMapDataType dt = kBF16) {
  EncodeTiledFn f = encode_fn();
  if (!f || !base) return false;
  cuuint64_t dims[3] = {cols, rows, z};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {64, box_rows, box_z};
  cuuint32_t es[3] = {1, 1, 1};
  return f(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 map of rank 3 or 4 with explicit strides (bytes, dims 1..rank-1) and box.
bool map_nd(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
            const uint32_t* box) {
  EncodeTiledFn f = encode_fn();
  if (!f || !base || rank < 3 || rank > 4) return false;
  cuuint64_t d[4], st[3];
  cuuint32_t b[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides[i];
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), d, st, b, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of a row-major [rows][cols] bf16 matrix as (64 columns, rows, cols/64 chunks) with
// strides (row, 128 B): a box of (64, box_rows, 2) is two consecutive 64-wide k chunks.
bool map_kpair(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[3] = {64, rows, cols / 64};
  const uint64_t strides[2] = {cols * 2, 128};
  const uint32_t box[3] = {64, box_rows, 2};
  return map_nd(m, base, 3, dims, strides, box);
}

// An activation in two planes [2][rows][cols] (hi, then lo), as (64 columns, rows, plane): a box
// of (64, box_rows, 2) is one 64-wide k chunk of both planes.
bool map_planes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[3] = {cols, rows, 2};
  const uint64_t strides[2] = {cols * 2, cols * rows * 2};
  const uint32_t box[3] = {64, box_rows, 2};
  return map_nd(m, base, 3, dims, strides, box);
}

// The same as (64 columns, rows, plane, cols/64 chunks): a box of (64, box_rows, 2, 2) is two
// consecutive 64-wide k chunks of both planes, laid out [chunk][plane][row][64], so that per
// chunk the hi rows and then the lo rows form one MMA operand of 2 box_rows rows.
bool map_kpair_planes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[4] = {64, rows, 2, cols / 64};
  const uint64_t strides[3] = {cols * 2, cols * rows * 2, 128};
  const uint32_t box[4] = {64, box_rows, 2, 2};
  return map_nd(m, base, 4, dims, strides, box);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int round_up(int x, int a) { return (x + a - 1) / a * a; }
int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

constexpr size_t kSmemLimit = 232448;  // opt-in shared memory per CTA on sm_100

// Programmatic dependent launch for every kernel: a kernel may begin its prologue and
// weight loads while its predecessor drains; its griddepcontrol.wait orders everything else.

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// plan
// ---------------------------------------------------------------------------
constexpr uint64_t kPlanMagic = 0x4F52544852555331ull;  // "ORTHRUS1"
constexpr int kMaxDraftSteps = 8;  // denoising steps of the draft view per decode step

struct LayerPtrs {
  const float *attn_norm, *mlp_norm, *q_norm, *k_norm, *wd_q_norm, *wd_k_norm;
  const void *w_qkv, *w_o, *w_gu, *w_down, *wd_qkv, *wd_o;
};

struct alignas(64) Plan {
  uint64_t magic;
  orthrus_config cfg;
  int L, B, cap, max_block, max_rows, sms, chunk_keys, attn_slots;
  const void* embed;
  const float* final_norm;
  const void* lm_head;
  __half *kc, *vc;  // bf16 values in the fp16 encoding
  int* len;
  void* ws;
  size_t ws_bytes;
  int* status;
  float* h;
  __nv_bfloat16 *xn, *attn, *act;  // [2][rows][cols]: hi plane, lo plane at + *_lo elements
  size_t xn_lo, attn_lo, act_lo;
  __half *qbuf, *blk_k, *blk_v;
  float2* rope;
  unsigned long long* amax;
  int *draft_ids, *ar_ids;
  float2* samp;     // per-row (max, normaliser) of the sampling kernels: [B * (2 max_block + 1)]
  float* samp_tot;  // per-row CDF tile totals: [B * max_block][kSampMaxTiles]
  float* gemm_part;
  int* gemm_cnt;
  float* att_o;
  float2* att_ml;
  int* att_cnt;
  // persistent forward kernel
  CUtensorMap* d_maps;  // device copy of the tensor maps
  LayerNorms* d_norms;  // device copy of the per-layer gains
  int* phase_cnt;
  int* exit_cnt;
  float* ss;
  int ss_ld, mega_slots, fwd_ck;
  float* fwd_att_o;
  float2* fwd_att_ml;
  size_t layers_off, maps_off, norms_off;
  // profiling hook (host memory, written during the calls)
  void* const* trace_ev;
  int32_t* trace_kind;
  int32_t trace_cap;
  int32_t* trace_count;
  unsigned long long* timeline;  // device, nullable: per-CTA phase events of the persistent kernel
  size_t timeline_bytes;

  const LayerPtrs& layer(int l) const { return reinterpret_cast<const LayerPtrs*>((const char*)this + layers_off)[l]; }
  LayerPtrs& layer(int l) { return reinterpret_cast<LayerPtrs*>((char*)this + layers_off)[l]; }
  const CUtensorMap& lmap(int l, int which) const {
    return reinterpret_cast<const CUtensorMap*>((const char*)this + maps_off)[l * M_PER_LAYER + which];
  }
  CUtensorMap* lmap_mut(int l, int which) {
    return reinterpret_cast<CUtensorMap*>((char*)this + maps_off) + l * M_PER_LAYER + which;
  }
  LayerNorms* norms_host() { return reinterpret_cast<LayerNorms*>((char*)this + norms_off); }
  const CUtensorMap& gmap(int which) const {
    return reinterpret_cast<const CUtensorMap*>((const char*)this + maps_off)[L * M_PER_LAYER + which];
  }
  CUtensorMap* gmap_mut(int which) {
    return reinterpret_cast<CUtensorMap*>((char*)this + maps_off) + L * M_PER_LAYER + which;
  }
};

size_t n_maps(int L) { return (size_t)L * M_PER_LAYER + G_COUNT; }

size_t plan_layout(int L, size_t* layers_off, size_t* maps_off, size_t* norms_off) {
  size_t off = align_up(sizeof(Plan), 64);
  *layers_off = off;
  off = align_up(off + sizeof(LayerPtrs) * (size_t)L, 64);
  *maps_off = off;
  off = align_up(off + sizeof(CUtensorMap) * n_maps(L), 64);
  *norms_off = off;
  off += sizeof(LayerNorms) * (size_t)L;
  return off + 64;  // slack for aligning the caller's buffer
}

Plan* plan_cast(const void* p) {
  if (!p) return nullptr;
  Plan* P = (Plan*)(((uintptr_t)p + 63) & ~(uintptr_t)63);
  return P->magic == kPlanMagic ? P : nullptr;
}

bool config_ok(const orthrus_config* c) {
  if (!c) return false;
  if (c->n_layers < 1 || c->d_model < 128 || c->n_heads < 1 || c->n_kv_heads < 1) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->n_heads % c->n_kv_heads) return false;
  const int G = c->n_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (c->d_model % 128 || c->d_ff % 128 || (c->n_heads * c->head_dim) % 128 || c->vocab % 128) return false;
  if (((c->n_heads + 2 * c->n_kv_heads) * c->head_dim) % 128) return false;
  if (c->mask_id < 0 || c->mask_id >= c->vocab) return false;
  return true;
}

// Split-KV chunk size for a cache of `cap` keys: chunk boundaries sit at fixed
// absolute positions for every call made with the same (batch, capacity).
int attn_chunk_keys(int B, int Hkv, int row_tiles, int cap) {
  const int sms = num_sms();
  const int units = std::max(1, B * Hkv * row_tiles);
  const int target = std::max(1, (2 * sms + units - 1) / units);
  return round_up(std::max(128, (cap + target - 1) / target), 128);
}

// workspace layout
struct WsLayout {
  size_t status, h, xn, qbuf, attn, act, rope, amax, draft_ids, ar_ids, samp, samp_tot, gemm_part, gemm_cnt, att_o, att_ml, att_cnt,
      blk_k, blk_v, dev_maps, dev_norms, phase_cnt, ss, fwd_att_o, fwd_att_ml, total;
  int chunk_keys, attn_slots, ss_ld, mega_slots;
};

bool fwd_rows_fit(int M, int d);

// Largest block (token rows per sequence, at most max_block + 1) whose B rows the persistent
// forward kernel runs; 0 if none. Larger blocks of the same plan take the per-op kernels.
int persistent_q_max(const orthrus_config* c, int B, int max_block) {
  for (int Q = max_block + 1; Q >= 1; --Q)
    if (fwd_rows_fit(B * Q, c->head_dim)) return Q;
  return 0;
}

// Attention slots of the persistent forward kernel for this batch and block limit
// (0 when the kernel runs no block of this plan: too many token rows or too many slots).
int mega_slots(const orthrus_config* c, int B, int max_block) {
  const int G = c->n_heads / c->n_kv_heads;
  const int qp = persistent_q_max(c, B, max_block);
  if (qp == 0 || c->d_model > 8192) return 0;
  const int rt = (G * qp + 127) / 128;
  const int slots = B * c->n_kv_heads * rt;
  return slots <= kMaxSlots ? slots : 0;
}

int gemm_counter_count(const orthrus_config* c, int max_rows) {
  const int mt = (max_rows + 127) / 128;
  int nt = std::max({c->vocab / 128, c->d_ff / 64, ((c->n_heads + 2 * c->n_kv_heads) * c->head_dim) / 128,
                     c->d_model / 128});
  return mt * nt;
}

// Rows allocated for activation buffers: a multiple of 128 so that any token tile fits.
int act_rows(int max_rows) { return round_up(std::max(max_rows, 128), 128); }

WsLayout ws_layout(const orthrus_config* c, int B, int max_block, int max_rows_req, int cap) {
  WsLayout w{};
  const int max_rows = act_rows(max_rows_req);
  const int D = c->d_model, Hd = c->n_heads * c->head_dim, F = c->d_ff, d = c->head_dim, L = c->n_layers;
  const int G = c->n_heads / c->n_kv_heads, Hkv = c->n_kv_heads;
  const int sms = num_sms();
  const int rt_dec = (G * (max_block + 1) + 127) / 128;
  const int ck = attn_chunk_keys(B, Hkv, rt_dec, cap);
  w.chunk_keys = ck;
  const int max_chunks = (cap + ck - 1) / ck + 1;
  const int rt_pre = (G * max_rows_req + 127) / 128;
  w.attn_slots = std::max(B * Hkv * rt_dec, Hkv * rt_pre) * max_chunks;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.status = take(256);
  w.h = take((size_t)max_rows * D * 4);
  w.xn = take((size_t)2 * max_rows * D * 2);  // hi and lo planes
  w.qbuf = take((size_t)max_rows * Hd * 2 + 128 * d * 2);
  w.attn = take((size_t)2 * max_rows * Hd * 2);
  w.act = take((size_t)2 * max_rows * F * 2);
  w.rope = take((size_t)max_rows * (d / 2) * 8);
  w.amax = take((size_t)max_rows * 8);
  w.draft_ids = take((size_t)B * max_block * 4);
  w.ar_ids = take((size_t)B * (max_block + 1) * 4);
  w.samp = take((size_t)B * (2 * max_block + 1) * 8);
  w.samp_tot = take((size_t)B * max_block * kSampMaxTiles * 4);
  w.gemm_part = take((size_t)2 * sms * 128 * 128 * 4);
  w.gemm_cnt = take((size_t)gemm_counter_count(c, max_rows) * 4);
  w.att_o = take((size_t)w.attn_slots * 128 * d * 4);
  w.att_ml = take((size_t)w.attn_slots * 128 * 8);
  w.att_cnt = take((size_t)std::max(B * Hkv * rt_dec, Hkv * rt_pre) * 4);
  const size_t blk = (size_t)L * B * Hkv * max_block * d * 2;
  w.blk_k = take(blk);
  w.blk_v = take(blk);
  w.dev_maps = take(sizeof(CUtensorMap) * ((size_t)L * M_PER_LAYER + G_COUNT));
  w.dev_norms = take(sizeof(LayerNorms) * (size_t)L);
  w.phase_cnt = take((size_t)(fwd_n_phases(L) + 1) * 4);
  w.ss_ld = max_rows;
  w.ss = take((size_t)(D / 128) * max_rows * 4);
  w.mega_slots = mega_slots(c, B, max_block);
  w.fwd_att_o = take((size_t)std::max(1, w.mega_slots) * kMaxChunks * 128 * d * 4);
  w.fwd_att_ml = take((size_t)std::max(1, w.mega_slots) * kMaxChunks * 128 * 8);
  w.total = off;
  return w;
}

template <typename F>
bool set_smem_attr(F* kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
}

// The dynamic shared-memory opt-in is a property of (kernel, device): it is set once per
// pair, under a lock, so that host threads and calls on a second GPU each get it.
template <typename F>
bool ensure_smem_attr(F* kernel, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<int, const void*>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const std::pair<int, const void*> key(dev, (const void*)kernel);
  std::lock_guard<std::mutex> lock(mu);
  if (std::find(done.begin(), done.end(), key) != done.end()) return true;
  if (!set_smem_attr(kernel, bytes)) return false;
  done.push_back(key);
  return true;
}

// ---------------------------------------------------------------------------
// launches
// ---------------------------------------------------------------------------
template <int EPI>
cudaError_t launch_gemm(const CUtensorMap& tmW, const CUtensorMap& tmX, GemmArgs a, int N, int Kd, int M,
                        cudaStream_t st) {
  a.N = N;
  a.Kd = Kd;
  a.M = M;
  a.m_tiles = (M + 127) / 128;
  a.Mt = a.m_tiles > 1 ? 128 : round_up(std::max(M, 1), 16);
  a.planes = std::max(1, a.planes);
  a.mt_alloc = std::max(32, next_pow2(a.planes * a.Mt));  // hi and lo products side by side
  a.n_tiles = (EPI == EPI_SWIGLU) ? N / 128 : N / 128;  // SwiGLU: N = 2F, a tile = 64 gate + 64 up rows
  a.k_chunks = Kd / 64;
  a.total_units = (long long)a.m_tiles * a.n_tiles * a.k_chunks;
  const int G = (int)std::min<long long>(num_sms(), a.total_units);
  const size_t fixed = gemm_smem_bytes(a.Mt, 0, a.planes);
  const size_t stage = 16384 + (size_t)a.Mt * 128 * a.planes;
  a.stages = (int)std::min<size_t>(12, (kSmemLimit - fixed) / stage);
  const size_t smem = gemm_smem_bytes(a.Mt, a.stages, a.planes);
  if (!ensure_smem_attr(gemm_kernel<EPI>, kSmemLimit)) return cudaErrorInvalidValue;
  return launch(gemm_kernel<EPI>, dim3(G), dim3(kGemmThreads), smem, st, tmW, tmX, a);
}

cudaError_t launch_attention(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tkb, const CUtensorMap& tvb, const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.max_chunks, a.row_tiles, a.B * a.Hkv);
  const size_t smem = attn_smem_bytes(d);
  if (d == 128) {
    if (!ensure_smem_attr(attention_kernel<128>, kSmemLimit)) return cudaErrorInvalidValue;
    return launch(attention_kernel<128>, grid, dim3(kAttnThreads), smem, st, tq, tk, tv, tkb, tvb, a);
  } else {
    if (!ensure_smem_attr(attention_kernel<64>, kSmemLimit)) return cudaErrorInvalidValue;
    return launch(attention_kernel<64>, grid, dim3(kAttnThreads), smem, st, tq, tk, tv, tkb, tvb, a);
  }
}

void mark(const Plan* P, int kind, cudaStream_t st) {
  if (!P->trace_ev || !P->trace_count) return;
  const int i = *P->trace_count;
  if (i >= P->trace_cap) return;
  cudaEventRecord((cudaEvent_t)P->trace_ev[i], st);
  P->trace_kind[i] = kind;
  *P->trace_count = i + 1;
}

// token-tile height of a GEMM over M rows (must match launch_gemm) -> map index
int mt_index(int M) {
  const int Mt = M > 128 ? 128 : round_up(std::max(M, 1), 16);
  return Mt / 16 - 1;
}

GemmArgs base_gemm_args(const Plan* P) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.partial = P->gemm_part;
  a.tile_counter = P->gemm_cnt;
  a.status = P->status;
  a.planes = 2;  // layer projections read both activation planes
  return a;
}

// ---------------------------------------------------------------------------
// persistent forward kernel (draft and verify views, at most 128 token rows)
// ---------------------------------------------------------------------------
// Blocks whose token rows fit two ring stages (at most 96 rows at head_dim 128) run through
// it; larger blocks take the per-op kernels.
bool fwd_rows_fit(int M, int d) {
  return M <= 128 && fwd_fixed_smem(d) + 2 * (size_t)fwd_stage_bytes(round_up(M, 16), d) <= kSmemLimit;
}

bool persistent_ok(const Plan* P, int Q) {
  return P->mega_slots > 0 && fwd_rows_fit(P->B * Q, P->cfg.head_dim) && Q <= P->max_block + 1;
}

template <int D, bool TL, bool G2>
cudaError_t launch_forward_inst(cudaLaunchConfig_t& cfg, const FwdArgs& a) {
  if (!ensure_smem_attr(forward_kernel<D, TL, G2>, kSmemLimit)) return cudaErrorInvalidValue;
  return cudaLaunchKernelEx(&cfg, forward_kernel<D, TL, G2>, a);
}

template <int D>
cudaError_t launch_forward_d(cudaLaunchConfig_t& cfg, const FwdArgs& a, bool tl, bool g2) {
  if (tl) return g2 ? launch_forward_inst<D, true, true>(cfg, a) : launch_forward_inst<D, true, false>(cfg, a);
  return g2 ? launch_forward_inst<D, false, true>(cfg, a) : launch_forward_inst<D, false, false>(cfg, a);
}

orthrus_status launch_forward(const Plan* P, int view, int Q, const int* pending, const int* draft, int* out_ids,
                              float* logits, bool accept, int K, int* pending_out, int* accept_len, int* committed,
                              cudaStream_t st) {
  const orthrus_config& c = P->cfg;
  FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.maps = P->d_maps;
  a.norms = P->d_norms;
  a.L = P->L;
  a.D = c.d_model;
  a.H = c.n_heads;
  a.Hkv = c.n_kv_heads;
  a.d = c.head_dim;
  a.F = c.d_ff;
  a.V = c.vocab;
  a.G = c.n_heads / c.n_kv_heads;
  a.qk_norm = c.qk_norm;
  a.mask_id = c.mask_id;
  a.eps = c.rms_eps;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c.head_dim));
  a.theta = (double)c.rope_theta;
  a.view = view;
  a.nb = P->B;
  a.Q = Q;
  a.M = P->B * Q;
  a.Mt = round_up(a.M, 16);
  a.mt_idx = a.Mt / 16 - 1;
  const size_t stage = fwd_stage_bytes(a.Mt, a.d);
  // 3-4 stages of 32 KB weight boxes (96-128 KB in flight per SM): a bare TMA stream of
  // such boxes measured fastest at 4; deeper rings put more requests in flight than HBM
  // serves efficiently
  a.stages = (int)std::min<size_t>(4, (kSmemLimit - fwd_fixed_smem(a.d)) / stage);
  a.stages = std::max(2, a.stages);
  const size_t smem = fwd_fixed_smem(a.d) + (size_t)a.stages * stage;
  a.cap = P->cap;
  a.max_block = P->max_block;
  a.batch = P->B;
  const int sms = num_sms();
  a.ck = P->fwd_ck;
  a.lookahead = 2;  // k-pair tiles of run-ahead past an unmet dependency: 2 measured best
  a.poll_ns = 64;   // sleep between polls of a phase counter
  a.pending = pending;
  a.draft_ids = draft;
  a.len = P->len;
  a.embed = (const __nv_bfloat16*)P->embed;
  a.final_norm = P->final_norm;
  a.kc = P->kc;
  a.vc = P->vc;
  a.blk_k = P->blk_k;
  a.blk_v = P->blk_v;
  a.h = P->h;
  a.xg = P->xn;
  a.qbuf = P->qbuf;
  a.attn = P->attn;
  a.act = P->act;
  a.xg_lo = P->xn_lo;
  a.attn_lo = P->attn_lo;
  a.act_lo = P->act_lo;
  a.rope = P->rope;
  a.ss = P->ss;
  a.ss_ld = P->ss_ld;
  a.amax = P->amax;
  a.out_ids = out_ids;
  a.logits = logits;
  a.partial = P->gemm_part;
  a.tile_cnt = P->gemm_cnt;
  a.phase_cnt = P->phase_cnt;
  a.exit_cnt = P->exit_cnt;
  a.att_o = P->fwd_att_o;
  a.att_ml = P->fwd_att_ml;
  a.status = P->status;
  a.diag = P->status + 16;  // inside the status block of the workspace
  const size_t tl_need = (size_t)num_sms() * fwd_n_phases(P->L) * TL_EVENTS * 8;
  a.tl = (P->timeline && P->timeline_bytes >= tl_need) ? P->timeline : nullptr;
  a.accept = accept ? 1 : 0;
  a.K = K;
  a.pending_out = pending_out;
  a.accept_len = accept_len;
  a.committed = committed;

  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kFwdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  // the timeline instantiation only while a timeline buffer is set (profiling); the G2 one for
  // blocks of 33-36 token rows (a K = 32 verify block)
  const bool g2 = a.M > 32 && a.M <= 36;
  if (c.head_dim == 128) e = launch_forward_d<128>(cfg, a, a.tl != nullptr, g2);
  else e = launch_forward_d<64>(cfg, a, a.tl != nullptr, g2);
  return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

// One forward over a block of Q rows for sequences [b0, b0+nb).
//   kind: BLOCK_DRAFT / BLOCK_VERIFY / BLOCK_PREFILL
//   head: run final norm + LM head + argmax; last_row_only: only row Q-1 of each sequence
//   argmax_out: [rows of the head] int32; logits: nullable fp32 [rows][vocab]
orthrus_status forward(const Plan* P, int kind, int b0, int nb, int Q, const int* pending, const int* draft,
                       const int* tokens, int tok_stride, int tok_off, bool head, bool last_row_only, int* argmax_out,
                       float* logits, cudaStream_t st) {
  const orthrus_config& c = P->cfg;
  const int D = c.d_model, H = c.n_heads, Hkv = c.n_kv_heads, d = c.head_dim, F = c.d_ff, V = c.vocab;
  const int G = H / Hkv, M = nb * Q;
  const bool draft_view = kind == BLOCK_DRAFT;

  EmbedArgs ea;
  ea.kind = kind;
  ea.nb = nb;
  ea.b0 = b0;
  ea.Q = Q;
  ea.D = D;
  ea.d = d;
  ea.V = V;
  ea.mask_id = c.mask_id;
  ea.cap = P->cap;
  ea.theta = (double)c.rope_theta;
  ea.pending = pending;
  ea.draft = draft;
  ea.tokens = tokens;
  ea.tok_stride = tok_stride;
  ea.tok_off = tok_off;
  ea.len = P->len;
  ea.embed = (const __nv_bfloat16*)P->embed;
  ea.h = P->h;
  ea.rope = P->rope;
  ea.status = P->status;
  mark(P, ORTHRUS_KIND_EMBED, st);
  if (launch(embed_kernel, dim3(M), dim3(256), 0, st, ea) != cudaSuccess) return ORTHRUS_ERR_CUDA;

  AttnArgs aa;
  memset(&aa, 0, sizeof(aa));
  aa.B = nb;
  aa.Hkv = Hkv;
  aa.G = G;
  aa.Q = Q;
  aa.d = d;
  aa.mode = draft_view ? 0 : 1;
  aa.b0 = b0;
  aa.rows = Q * G;
  aa.row_tiles = (aa.rows + 127) / 128;
  aa.chunk_keys = P->chunk_keys;
  aa.cap = P->cap;
  aa.max_chunks = (P->cap + P->chunk_keys - 1) / P->chunk_keys + (draft_view ? 1 : 0);
  aa.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
  aa.len = P->len;
  aa.out = P->attn;
  aa.out_lo = P->attn_lo;
  aa.part_o = P->att_o;
  aa.part_ml = P->att_ml;
  aa.counter = P->att_cnt;
  aa.status = P->status;
  if ((long long)nb * Hkv * aa.row_tiles * aa.max_chunks > P->attn_slots) return ORTHRUS_ERR_WORKSPACE;

  for (int l = 0; l < P->L; ++l) {
    const LayerPtrs& lp = P->layer(l);
    mark(P, ORTHRUS_KIND_RMSNORM, st);
    if (launch(rmsnorm_kernel, dim3(M), dim3(256), 0, st, (const float*)P->h, D, lp.attn_norm, c.rms_eps, P->xn,
               P->xn_lo, 0, 1, (unsigned long long*)nullptr) != cudaSuccess)
      return ORTHRUS_ERR_CUDA;

    GemmArgs g = base_gemm_args(P);
    g.qkv.H = H;
    g.qkv.Hkv = Hkv;
    g.qkv.d = d;
    g.qkv.Q = Q;
    g.qkv.b0 = b0;
    g.qkv.qk_norm = c.qk_norm;
    g.qkv.mode = draft_view ? VIEW_DRAFT : VIEW_VERIFY;
    g.qkv.eps = c.rms_eps;
    g.qkv.gq = draft_view ? lp.wd_q_norm : lp.q_norm;
    g.qkv.gk = draft_view ? lp.wd_k_norm : lp.k_norm;
    g.qkv.rope = P->rope;
    g.qkv.len = P->len;
    g.qkv.qbuf = P->qbuf;
    if (draft_view) {
      const size_t lo = (size_t)l * P->B * Hkv * P->max_block * d;
      g.qkv.kdst = P->blk_k + lo;
      g.qkv.vdst = P->blk_v + lo;
      g.qkv.kv_stride = P->max_block;
    } else {
      const size_t lo = (size_t)l * P->B * Hkv * P->cap * d;
      g.qkv.kdst = P->kc + lo;
      g.qkv.vdst = P->vc + lo;
      g.qkv.kv_stride = P->cap;
    }
    const int qkv_rows = (H + 2 * Hkv) * d;
    mark(P, ORTHRUS_KIND_GEMM_QKV, st);
    if ((launch_gemm<EPI_QKV>(P->lmap(l, draft_view ? M_WDQKV : M_WQKV), P->gmap(G_XNP + mt_index(M)), g, qkv_rows, D, M, st)) !=
        cudaSuccess)
      return ORTHRUS_ERR_CUDA;

    aa.z_cache = l * P->B * Hkv;
    aa.z_blk = l * P->B * Hkv;
    mark(P, ORTHRUS_KIND_ATTENTION, st);
    if ((launch_attention(d, P->gmap(G_Q), P->gmap(G_KC), P->gmap(G_VC), P->gmap(G_KB), P->gmap(G_VB), aa, st)) !=
        cudaSuccess)
      return ORTHRUS_ERR_CUDA;

    g = base_gemm_args(P);
    g.out_f32 = P->h;
    g.ld_out = D;
    mark(P, ORTHRUS_KIND_GEMM_O, st);
    if ((launch_gemm<EPI_RESID>(P->lmap(l, draft_view ? M_WDO : M_WO), P->gmap(G_ATTN + mt_index(M)), g, D, H * d, M, st)) !=
        cudaSuccess)
      return ORTHRUS_ERR_CUDA;

    mark(P, ORTHRUS_KIND_RMSNORM, st);
    if (launch(rmsnorm_kernel, dim3(M), dim3(256), 0, st, (const float*)P->h, D, lp.mlp_norm, c.rms_eps, P->xn,
               P->xn_lo, 0, 1, (unsigned long long*)nullptr) != cudaSuccess)
      return ORTHRUS_ERR_CUDA;
    g = base_gemm_args(P);
    g.out_bf16 = P->act;
    g.out_lo = P->act_lo;
    g.ld_out = F;
    g.swiglu_F = F;
    mark(P, ORTHRUS_KIND_GEMM_GATE_UP, st);
    if ((launch_gemm<EPI_SWIGLU>(P->lmap(l, M_WGU), P->gmap(G_XNP + mt_index(M)), g, 2 * F, D, M, st)) != cudaSuccess)
      return ORTHRUS_ERR_CUDA;

    g = base_gemm_args(P);
    g.out_f32 = P->h;
    g.ld_out = D;
    mark(P, ORTHRUS_KIND_GEMM_DOWN, st);
    if ((launch_gemm<EPI_RESID>(P->lmap(l, M_WDOWN), P->gmap(G_ACT + mt_index(M)), g, D, F, M, st)) != cudaSuccess)
      return ORTHRUS_ERR_CUDA;
  }

  if (!head) return cudaGetLastError() == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
  const int HR = last_row_only ? nb : M;
  mark(P, ORTHRUS_KIND_RMSNORM, st);
  if (launch(rmsnorm_kernel, dim3(HR), dim3(256), 0, st, (const float*)P->h, D, P->final_norm, c.rms_eps, P->xn,
             (size_t)0, last_row_only ? Q - 1 : 0, last_row_only ? Q : 1, P->amax) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  GemmArgs g = base_gemm_args(P);
  g.planes = 1;  // the LM head reads the hi plane only
  g.amax = P->amax;
  g.logits = logits;
  g.ld_logits = V;
  mark(P, ORTHRUS_KIND_LM_HEAD, st);
  if ((launch_gemm<EPI_ARGMAX>(P->gmap(G_LM), P->gmap(G_XN + mt_index(HR)), g, V, D, HR, st)) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  mark(P, ORTHRUS_KIND_ARGMAX, st);
  if (launch(argmax_finalize_kernel, dim3((HR + 127) / 128), dim3(128), 0, st, (const unsigned long long*)P->amax, HR,
             argmax_out, P->status) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

size_t orthrus_plan_bytes(const orthrus_config* cfg) {
  if (!config_ok(cfg)) return 0;
  size_t a, b, n;
  return plan_layout(cfg->n_layers, &a, &b, &n);
}

static bool sizes_ok(const orthrus_config* cfg, int batch, int capacity, int max_block, int max_rows) {
  return config_ok(cfg) && batch >= 1 && capacity >= 1 && max_block >= 1 && max_block <= 64 &&
         (long long)max_rows >= (long long)batch * (max_block + 1) && max_rows <= (1 << 20);
}

size_t orthrus_workspace_bytes(const orthrus_config* cfg, int32_t batch, int32_t capacity, int32_t max_block,
                               int32_t max_rows) {
  if (!sizes_ok(cfg, batch, capacity, max_block, max_rows)) return 0;
  return ws_layout(cfg, batch, max_block, max_rows, capacity).total;
}

size_t orthrus_block_scratch_offset(const orthrus_config* cfg, int32_t batch, int32_t capacity, int32_t max_block,
                                    int32_t max_rows) {
  if (!sizes_ok(cfg, batch, capacity, max_block, max_rows)) return 0;
  return ws_layout(cfg, batch, max_block, max_rows, capacity).blk_k;
}

size_t orthrus_block_scratch_bytes(const orthrus_config* cfg, int32_t batch, int32_t max_block) {
  if (!config_ok(cfg) || batch < 1 || max_block < 1) return 0;
  return 2ull * cfg->n_layers * batch * max_block * cfg->n_kv_heads * cfg->head_dim * 2ull;
}

orthrus_status orthrus_plan_init(void* plan, size_t plan_bytes, const orthrus_config* cfg, const orthrus_weights* w,
                                 const orthrus_cache* cache, int32_t max_block, int32_t max_rows, void* workspace,
                                 size_t workspace_bytes, orthrus_stream stream) {
  if (!plan || !cfg || !w || !cache || !workspace) return ORTHRUS_ERR_ARG;
  if (!config_ok(cfg)) return ORTHRUS_ERR_UNSUPPORTED;
  if (!cache->k || !cache->v || !cache->len) return ORTHRUS_ERR_ARG;
  if (!sizes_ok(cfg, cache->batch, cache->capacity, max_block, max_rows)) return ORTHRUS_ERR_ARG;
  const int L = cfg->n_layers;
  size_t layers_off, maps_off, norms_off;
  if (plan_bytes < plan_layout(L, &layers_off, &maps_off, &norms_off)) return ORTHRUS_ERR_WORKSPACE;
  const WsLayout wl = ws_layout(cfg, cache->batch, max_block, max_rows, cache->capacity);
  if (workspace_bytes < wl.total) return ORTHRUS_ERR_WORKSPACE;
  if (!w->embed || !w->final_norm || !w->lm_head || !w->attn_norm || !w->mlp_norm || !w->w_qkv || !w->w_o ||
      !w->w_gate_up || !w->w_down || !w->wd_qkv || !w->wd_o)
    return ORTHRUS_ERR_ARG;
  if (cfg->qk_norm && (!w->q_norm || !w->k_norm || !w->wd_q_norm || !w->wd_k_norm)) return ORTHRUS_ERR_ARG;
  if (!encode_fn()) return ORTHRUS_ERR_CUDA;

  Plan* P = (Plan*)(((uintptr_t)plan + 63) & ~(uintptr_t)63);
  memset(P, 0, sizeof(Plan));
  P->cfg = *cfg;
  P->L = L;
  P->B = cache->batch;
  P->cap = cache->capacity;
  P->max_block = max_block;
  P->max_rows = max_rows;
  P->sms = num_sms();
  P->chunk_keys = wl.chunk_keys;
  P->attn_slots = wl.attn_slots;
  P->embed = w->embed;
  P->final_norm = w->final_norm;
  P->lm_head = w->lm_head;
  P->kc = (__half*)cache->k;
  P->vc = (__half*)cache->v;
  P->len = cache->len;
  P->ws = workspace;
  P->ws_bytes = workspace_bytes;
  char* base = (char*)workspace;
  P->status = (int*)(base + wl.status);
  P->h = (float*)(base + wl.h);
  P->xn = (__nv_bfloat16*)(base + wl.xn);
  P->qbuf = (__half*)(base + wl.qbuf);
  P->attn = (__nv_bfloat16*)(base + wl.attn);
  P->act = (__nv_bfloat16*)(base + wl.act);
  {
    const size_t r = (size_t)act_rows(max_rows);
    P->xn_lo = r * cfg->d_model;
    P->attn_lo = r * cfg->n_heads * cfg->head_dim;
    P->act_lo = r * cfg->d_ff;
  }
  P->rope = (float2*)(base + wl.rope);
  P->amax = (unsigned long long*)(base + wl.amax);
  P->draft_ids = (int*)(base + wl.draft_ids);
  P->ar_ids = (int*)(base + wl.ar_ids);
  P->samp = (float2*)(base + wl.samp);
  P->samp_tot = (float*)(base + wl.samp_tot);
  P->gemm_part = (float*)(base + wl.gemm_part);
  P->gemm_cnt = (int*)(base + wl.gemm_cnt);
  P->att_o = (float*)(base + wl.att_o);
  P->att_ml = (float2*)(base + wl.att_ml);
  P->att_cnt = (int*)(base + wl.att_cnt);
  P->blk_k = (__half*)(base + wl.blk_k);
  P->blk_v = (__half*)(base + wl.blk_v);
  P->d_maps = (CUtensorMap*)(base + wl.dev_maps);
  P->d_norms = (LayerNorms*)(base + wl.dev_norms);
  P->phase_cnt = (int*)(base + wl.phase_cnt);
  P->exit_cnt = P->phase_cnt + fwd_n_phases(L);
  P->ss = (float*)(base + wl.ss);
  P->ss_ld = wl.ss_ld;
  P->mega_slots = wl.mega_slots;
  // attention chunk of the persistent kernel, fixed per plan (so verify rows and plain AR rows
  // see the same chunk boundaries): at most kMaxChunks - 2 chunks over the whole capacity, and
  // long enough that a full cache's verify-view units (sequence, KV head, row tile, chunk) fit
  // one wave of CTAs
  P->fwd_ck = std::max(64, round_up((P->cap + kMaxChunks - 3) / (kMaxChunks - 2), 64));
  {
    const int G = cfg->n_heads / cfg->n_kv_heads;
    const int qp = std::max(1, persistent_q_max(cfg, P->B, max_block));  // largest persistent block
    const int slots_v = P->B * cfg->n_kv_heads * ((G * qp + 127) / 128);
    const int sms = num_sms();
    const int per_slot = std::max(1, sms / std::max(1, slots_v));  // chunks per slot in one wave
    P->fwd_ck = std::max(P->fwd_ck, round_up((P->cap + per_slot - 1) / per_slot, 64));
  }
  P->fwd_att_o = (float*)(base + wl.fwd_att_o);
  P->fwd_att_ml = (float2*)(base + wl.fwd_att_ml);
  P->norms_off = norms_off;
  P->layers_off = layers_off;
  P->maps_off = maps_off;

  const int D = cfg->d_model, H = cfg->n_heads, Hkv = cfg->n_kv_heads, d = cfg->head_dim, F = cfg->d_ff;
  const int V = cfg->vocab, qkv_rows = (H + 2 * Hkv) * d;
  bool ok = true;
  for (int l = 0; l < L; ++l) {
    LayerPtrs& lp = P->layer(l);
    lp.attn_norm = w->attn_norm[l];
    lp.mlp_norm = w->mlp_norm[l];
    lp.q_norm = cfg->qk_norm ? w->q_norm[l] : nullptr;
    lp.k_norm = cfg->qk_norm ? w->k_norm[l] : nullptr;
    lp.wd_q_norm = cfg->qk_norm ? w->wd_q_norm[l] : nullptr;
    lp.wd_k_norm = cfg->qk_norm ? w->wd_k_norm[l] : nullptr;
    lp.w_qkv = w->w_qkv[l];
    lp.w_o = w->w_o[l];
    lp.w_gu = w->w_gate_up[l];
    lp.w_down = w->w_down[l];
    lp.wd_qkv = w->wd_qkv[l];
    lp.wd_o = w->wd_o[l];
    if (!lp.attn_norm || !lp.mlp_norm) ok = false;
    if (cfg->qk_norm && (!lp.q_norm || !lp.k_norm || !lp.wd_q_norm || !lp.wd_k_norm)) ok = false;
    ok = ok && map2d(P->lmap_mut(l, M_WQKV), lp.w_qkv, D, qkv_rows, 64, 128);
    ok = ok && map2d(P->lmap_mut(l, M_WO), lp.w_o, H * d, D, 64, 128);
    ok = ok && map2d(P->lmap_mut(l, M_WGU), lp.w_gu, D, 2 * F, 64, 64);
    ok = ok && map2d(P->lmap_mut(l, M_WDOWN), lp.w_down, F, D, 64, 128);
    ok = ok && map2d(P->lmap_mut(l, M_WDQKV), lp.wd_qkv, D, qkv_rows, 64, 128);
    ok = ok && map2d(P->lmap_mut(l, M_WDO), lp.wd_o, H * d, D, 64, 128);
    ok = ok && map_kpair(P->lmap_mut(l, M_WQKV3), lp.w_qkv, D, qkv_rows, 128);
    ok = ok && map_kpair(P->lmap_mut(l, M_WO3), lp.w_o, H * d, D, 128);
    ok = ok && map_kpair(P->lmap_mut(l, M_WDOWN3), lp.w_down, F, D, 128);
    ok = ok && map_kpair(P->lmap_mut(l, M_WDQKV3), lp.wd_qkv, D, qkv_rows, 128);
    ok = ok && map_kpair(P->lmap_mut(l, M_WDO3), lp.wd_o, H * d, D, 128);
    {  // (64 columns, d_ff rows, gate|up half, k chunk)
      const uint64_t dims[4] = {64, (uint64_t)F, 2, (uint64_t)D / 64};
      const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)F * D * 2, 128};
      const uint32_t box[4] = {64, 64, 2, 2};
      ok = ok && map_nd(P->lmap_mut(l, M_WGU4), lp.w_gu, 4, dims, strides, box);
    }
    // the forward kernel reads norm gains as 16-byte vectors
    auto a16 = [](const void* q) { return q != nullptr && ((uintptr_t)q & 15u) == 0; };
    ok = ok && a16(lp.attn_norm) && a16(lp.mlp_norm) && a16(w->final_norm);
    ok = ok && (!cfg->qk_norm || (a16(lp.q_norm) && a16(lp.k_norm) && a16(lp.wd_q_norm) && a16(lp.wd_k_norm)));
    LayerNorms& ln = P->norms_host()[l];
    ln.attn_norm = lp.attn_norm;
    ln.mlp_norm = lp.mlp_norm;
    ln.q_norm = lp.q_norm;
    ln.k_norm = lp.k_norm;
    ln.wd_q_norm = lp.wd_q_norm;
    ln.wd_k_norm = lp.wd_k_norm;
  }
  ok = ok && map2d(P->gmap_mut(G_LM), w->lm_head, D, V, 64, 128);
  ok = ok && map_kpair(P->gmap_mut(G_LM3), w->lm_head, D, V, 128);
  const int rows = act_rows(max_rows);
  for (int i = 0; i < 8; ++i) {
    const uint32_t br = 16 * (i + 1);
    ok = ok && map2d(P->gmap_mut(G_XN + i), P->xn, D, rows, 64, br);  // hi plane only
    ok = ok && map_planes(P->gmap_mut(G_XNP + i), P->xn, D, rows, br);
    ok = ok && map_planes(P->gmap_mut(G_ATTN + i), P->attn, H * d, rows, br);
    ok = ok && map_planes(P->gmap_mut(G_ACT + i), P->act, F, rows, br);
    ok = ok && map_kpair(P->gmap_mut(G_XN3 + i), P->xn, D, rows, br);  // hi plane only
    ok = ok && map_kpair_planes(P->gmap_mut(G_XN4 + i), P->xn, D, rows, br);
    ok = ok && map_kpair_planes(P->gmap_mut(G_ATTN4 + i), P->attn, H * d, rows, br);
    ok = ok && map_kpair_planes(P->gmap_mut(G_ACT4 + i), P->act, F, rows, br);
  }
  ok = ok && map2d(P->gmap_mut(G_Q), P->qbuf, d, (uint64_t)rows * H + 128, 64, 128, kF16);
  const uint64_t zc = (uint64_t)L * P->B * Hkv;
  ok = ok && map3d(P->gmap_mut(G_KC), P->kc, d, P->cap, zc, 128, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_VC), P->vc, d, P->cap, zc, 128, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_KB), P->blk_k, d, max_block, zc, 128, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_VB), P->blk_v, d, max_block, zc, 128, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_KC64), P->kc, d, P->cap, zc, 64, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_VC64), P->vc, d, P->cap, zc, 64, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_KB64), P->blk_k, d, max_block, zc, 64, 1, kF16);
  ok = ok && map3d(P->gmap_mut(G_VB64), P->blk_v, d, max_block, zc, 64, 1, kF16);
  if (!ok) return ORTHRUS_ERR_ARG;
  if (cudaMemsetAsync(workspace, 0, wl.total, (cudaStream_t)stream) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  // the persistent kernel reads the tensor maps and norm gains from device memory
  if (cudaMemcpyAsync(P->d_maps, &P->lmap(0, 0), sizeof(CUtensorMap) * n_maps(L), cudaMemcpyHostToDevice,
                      (cudaStream_t)stream) != cudaSuccess ||
      cudaMemcpyAsync(P->d_norms, P->norms_host(), sizeof(LayerNorms) * L, cudaMemcpyHostToDevice,
                      (cudaStream_t)stream) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  P->magic = kPlanMagic;
  return ORTHRUS_OK;
}

int32_t* orthrus_status_ptr(const void* plan) {
  const Plan* P = plan_cast(plan);
  return P ? P->status : nullptr;
}

orthrus_status orthrus_clear_status(const void* plan, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P) return ORTHRUS_ERR_ARG;
  return cudaMemsetAsync(P->status, 0, sizeof(int), (cudaStream_t)stream) == cudaSuccess ? ORTHRUS_OK
                                                                                       : ORTHRUS_ERR_CUDA;
}

orthrus_status orthrus_trace(void* plan, void* const* events, int32_t* kinds, int32_t capacity, int32_t* count) {
  Plan* P = plan_cast(plan);
  if (!P) return ORTHRUS_ERR_ARG;
  if (!events) {
    P->trace_ev = nullptr;
    P->trace_kind = nullptr;
    P->trace_count = nullptr;
    P->trace_cap = 0;
    return ORTHRUS_OK;
  }
  if (!kinds || !count || capacity < 1) return ORTHRUS_ERR_ARG;
  P->trace_ev = events;
  P->trace_kind = kinds;
  P->trace_cap = capacity;
  P->trace_count = count;
  return ORTHRUS_OK;
}

size_t orthrus_timeline_bytes(const void* plan) {
  const Plan* P = plan_cast(plan);
  return P ? (size_t)num_sms() * fwd_n_phases(P->L) * TL_EVENTS * 8 : 0;
}

orthrus_status orthrus_timeline(void* plan, void* device_buf, size_t bytes) {
  Plan* P = plan_cast(plan);
  if (!P) return ORTHRUS_ERR_ARG;
  if (device_buf && bytes < orthrus_timeline_bytes(plan)) return ORTHRUS_ERR_WORKSPACE;
  P->timeline = (unsigned long long*)device_buf;
  P->timeline_bytes = device_buf ? bytes : 0;
  return ORTHRUS_OK;
}

int32_t orthrus_decode_step_launches(const void* plan, int32_t K) {
  const Plan* P = plan_cast(plan);
  if (!P || K < 1 || K > P->max_block) return 0;
  if (persistent_ok(P, K) && persistent_ok(P, K + 1)) return 2;
  const int per_forward = 1 + 7 * P->L + 3;
  return 2 * per_forward + 1;
}

orthrus_status orthrus_prefill(const void* plan, const int32_t* tokens, const int32_t* prompt_len, int32_t max_prompt,
                               int32_t* pending, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !tokens || !prompt_len || !pending || max_prompt < 1) return ORTHRUS_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  for (int b = 0; b < P->B; ++b)
    if (prompt_len[b] < 1 || prompt_len[b] > max_prompt) return ORTHRUS_ERR_ARG;
  for (int b = 0; b < P->B; ++b)
    if (prompt_len[b] > P->cap) return ORTHRUS_ERR_CAPACITY;
  const int chunk = P->max_rows;
  for (int b = 0; b < P->B; ++b) {
    const int Pb = prompt_len[b];
    for (int c0 = 0; c0 < Pb; c0 += chunk) {
      const int Q = std::min(chunk, Pb - c0);
      const bool last = c0 + Q == Pb;
      mark(P, ORTHRUS_KIND_OTHER, st);
      if (launch(set_len_kernel, dim3(1), dim3(1), 0, st, P->len, b, c0) != cudaSuccess) return ORTHRUS_ERR_CUDA;
      orthrus_status s = forward(P, BLOCK_PREFILL, b, 1, Q, nullptr, nullptr, tokens, max_prompt, c0, last, true,
                                 pending + b, nullptr, st);
      if (s != ORTHRUS_OK) return s;
    }
    mark(P, ORTHRUS_KIND_OTHER, st);
    if (launch(set_len_kernel, dim3(1), dim3(1), 0, st, P->len, b, Pb) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  }
  mark(P, ORTHRUS_KIND_END, st);
  return cudaGetLastError() == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

orthrus_status orthrus_draft_block(const void* plan, const int32_t* pending, int32_t K, int32_t* draft, float* logits,
                                   orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !draft || K < 1 || K > P->max_block) return ORTHRUS_ERR_ARG;
  orthrus_status s;
  if (persistent_ok(P, K)) {
    mark(P, ORTHRUS_KIND_FORWARD, (cudaStream_t)stream);
    s = launch_forward(P, VIEW_DRAFT, K, pending, nullptr, draft, logits, false, 0, nullptr, nullptr, nullptr,
                       (cudaStream_t)stream);
  } else {
    s = forward(P, BLOCK_DRAFT, 0, P->B, K, pending, nullptr, nullptr, 0, 0, true, false, draft, logits,
                (cudaStream_t)stream);
  }
  mark(P, ORTHRUS_KIND_END, (cudaStream_t)stream);
  return s;
}

orthrus_status orthrus_verify_block(const void* plan, const int32_t* pending, const int32_t* draft, int32_t K,
                                    int32_t* ar_argmax, float* logits, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !ar_argmax || K < 0 || K > P->max_block || (K > 0 && !draft)) return ORTHRUS_ERR_ARG;
  orthrus_status s;
  if (persistent_ok(P, K + 1)) {
    mark(P, ORTHRUS_KIND_FORWARD, (cudaStream_t)stream);
    s = launch_forward(P, VIEW_VERIFY, K + 1, pending, draft, ar_argmax, logits, false, K, nullptr, nullptr, nullptr,
                       (cudaStream_t)stream);
  } else {
    s = forward(P, BLOCK_VERIFY, 0, P->B, K + 1, pending, draft, nullptr, 0, 0, true, false, ar_argmax, logits,
                (cudaStream_t)stream);
  }
  mark(P, ORTHRUS_KIND_END, (cudaStream_t)stream);
  return s;
}

orthrus_status orthrus_accept_commit(const void* plan, int32_t* pending, const int32_t* draft,
                                     const int32_t* ar_argmax, int32_t K, int32_t* accept_len, int32_t* committed,
                                     int32_t poison_dead, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !ar_argmax || !accept_len || !committed || K < 0 || K > P->max_block || (K > 0 && !draft))
    return ORTHRUS_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  mark(P, ORTHRUS_KIND_ACCEPT, st);
  if (launch(accept_kernel, dim3(P->B), dim3(96), 0, st, pending, draft, ar_argmax, K, accept_len, committed, P->len,
             (const int*)P->status) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  if (poison_dead) mark(P, ORTHRUS_KIND_OTHER, st);
  if (poison_dead)
    if (launch(poison_kernel, dim3(P->L * P->B * P->cfg.n_kv_heads), dim3(128), 0, st, P->kc, P->vc,
               (const int*)P->len, (const int*)accept_len, K, P->B, P->cfg.n_kv_heads, P->cap, P->cfg.head_dim) !=
        cudaSuccess)
      return ORTHRUS_ERR_CUDA;
  mark(P, ORTHRUS_KIND_END, st);
  return cudaGetLastError() == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

orthrus_status orthrus_draft_refine(const void* plan, const int32_t* pending, const int32_t* prev_draft, int32_t K,
                                    int32_t* draft, float* logits, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !prev_draft || !draft || K < 1 || K > P->max_block) return ORTHRUS_ERR_ARG;
  orthrus_status s;
  if (persistent_ok(P, K)) {
    mark(P, ORTHRUS_KIND_FORWARD, (cudaStream_t)stream);
    s = launch_forward(P, VIEW_DRAFT, K, pending, prev_draft, draft, logits, false, 0, nullptr, nullptr, nullptr,
                       (cudaStream_t)stream);
  } else {
    s = forward(P, BLOCK_DRAFT, 0, P->B, K, pending, prev_draft, nullptr, 0, 0, true, false, draft, logits,
                (cudaStream_t)stream);
  }
  mark(P, ORTHRUS_KIND_END, (cudaStream_t)stream);
  return s;
}

orthrus_status orthrus_decode_step_ex(const void* plan, int32_t* pending, int32_t K, int32_t draft_steps,
                                      const int32_t* planted, int32_t* accept_len, int32_t* committed,
                                      orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !accept_len || !committed || K < 1 || K > P->max_block || draft_steps < 1 ||
      draft_steps > kMaxDraftSteps)
    return ORTHRUS_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  orthrus_status s = orthrus_draft_block(plan, pending, K, P->draft_ids, nullptr, stream);
  for (int i = 1; s == ORTHRUS_OK && i < draft_steps; ++i)  // in place: the ids are read before any is written
    s = orthrus_draft_refine(plan, pending, P->draft_ids, K, P->draft_ids, nullptr, stream);
  if (s != ORTHRUS_OK) return s;
  if (planted) mark(P, ORTHRUS_KIND_OTHER, st);
  if (planted && cudaMemcpyAsync(P->draft_ids, planted, sizeof(int) * P->B * K, cudaMemcpyDeviceToDevice, st) !=
                     cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  if (persistent_ok(P, K + 1)) {  // verify view with the greedy consensus fused into its last CTA
    mark(P, ORTHRUS_KIND_FORWARD, st);
    s = launch_forward(P, VIEW_VERIFY, K + 1, pending, P->draft_ids, P->ar_ids, nullptr, true, K, pending, accept_len,
                       committed, st);
    mark(P, ORTHRUS_KIND_END, st);
    return s;
  }
  s = orthrus_verify_block(plan, pending, P->draft_ids, K, P->ar_ids, nullptr, stream);
  if (s != ORTHRUS_OK) return s;
  return orthrus_accept_commit(plan, pending, P->draft_ids, P->ar_ids, K, accept_len, committed, 0, stream);
}

orthrus_status orthrus_decode_step(const void* plan, int32_t* pending, int32_t K, const int32_t* planted,
                                   int32_t* accept_len, int32_t* committed, orthrus_stream stream) {
  return orthrus_decode_step_ex(plan, pending, K, 1, planted, accept_len, committed, stream);
}

// ---- decoding at temperature T > 0 ------------------------------------------

static bool temperature_ok(float t) { return t > 0.f && t < INFINITY; }

orthrus_status orthrus_sample_tokens(const float* logits, int32_t rows, int32_t vocab, float temperature,
                                     const float* uniforms, int32_t* out, int32_t* status, orthrus_stream stream) {
  if (rows < 0 || vocab < 1 || vocab > kSampTile * kSampMaxTiles || !temperature_ok(temperature)) return ORTHRUS_ERR_ARG;
  if (rows == 0) return ORTHRUS_OK;
  if (!logits || !uniforms || !out) return ORTHRUS_ERR_ARG;
  if (launch(sample_rows_kernel, dim3(rows), dim3(kSampThreads), 0, (cudaStream_t)stream, logits, (int)vocab,
             1.f / temperature, uniforms, (int*)out, (int*)status) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  return ORTHRUS_OK;
}

// The consensus of a sampled step: statistics of the verify rows (and of the draft rows unless
// the draws already computed them), tile totals of the last token's weights, draw and commit.
static orthrus_status sampled_consensus(const Plan* P, int32_t* pending, const int32_t* draft, const float* dl,
                                        const float* vl, int K, float temperature, const float* u_accept,
                                        const float* u_final, int32_t* accept_len, int32_t* committed,
                                        bool draft_stats_ready, cudaStream_t st) {
  const int B = P->B, V = P->cfg.vocab;
  const float inv_t = 1.f / temperature;
  mark(P, ORTHRUS_KIND_SAMPLE, st);
  const int skip = draft_stats_ready ? B * K : 0;  // rows whose statistics are already in place
  if (launch(row_stats_kernel, dim3(B * (2 * K + 1) - skip), dim3(kSampThreads), 0, st, dl, B * K - skip, vl, V,
             inv_t, P->samp + skip, P->status) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  ConsensusArgs c;
  c.pending = (int*)pending;
  c.draft = (const int*)draft;
  c.dl = dl;
  c.vl = vl;
  c.stats = P->samp;
  c.tot = P->samp_tot;
  c.u_acc = u_accept;
  c.u_fin = u_final;
  c.accept_len = (int*)accept_len;
  c.committed = (int*)committed;
  c.len = P->len;
  c.status = P->status;
  c.B = B;
  c.K = K;
  c.V = V;
  c.inv_t = inv_t;
  const int nt = (V + kSampTile - 1) / kSampTile;
  mark(P, ORTHRUS_KIND_ACCEPT, st);
  if (launch(consensus_totals_kernel, dim3(B, (nt + kTotTiles - 1) / kTotTiles), dim3(kTotThreads), 0, st, c) !=
      cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  if (launch(consensus_select_kernel, dim3(B), dim3(kTotThreads), 0, st, c) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  mark(P, ORTHRUS_KIND_END, st);
  return ORTHRUS_OK;
}

orthrus_status orthrus_accept_sample(const void* plan, int32_t* pending, const int32_t* draft,
                                     const float* draft_logits, const float* verify_logits, int32_t K,
                                     float temperature, const float* u_accept, const float* u_final,
                                     int32_t* accept_len, int32_t* committed, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !verify_logits || !u_final || !accept_len || !committed || K < 0 || K > P->max_block ||
      !temperature_ok(temperature) || P->cfg.vocab > kSampTile * kSampMaxTiles)
    return ORTHRUS_ERR_ARG;
  if (K > 0 && (!draft || !draft_logits || !u_accept)) return ORTHRUS_ERR_ARG;
  return sampled_consensus(P, pending, draft, draft_logits, verify_logits, K, temperature, u_accept, u_final,
                           accept_len, committed, false, (cudaStream_t)stream);
}

orthrus_status orthrus_decode_step_sampled(const void* plan, int32_t* pending, int32_t K, float temperature,
                                           const float* u_draft, const float* u_accept, const float* u_final,
                                           float* draft_logits, float* verify_logits, int32_t* accept_len,
                                           int32_t* committed, orthrus_stream stream) {
  const Plan* P = plan_cast(plan);
  if (!P || !pending || !u_draft || !u_accept || !u_final || !draft_logits || !verify_logits || !accept_len ||
      !committed || K < 1 || K > P->max_block || !temperature_ok(temperature) ||
      P->cfg.vocab > kSampTile * kSampMaxTiles)
    return ORTHRUS_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  orthrus_status s = orthrus_draft_block(plan, pending, K, P->draft_ids, draft_logits, stream);
  if (s != ORTHRUS_OK) return s;
  // the drafts: statistics of the draft rows, tile totals, draws (the indices orthrus_sample_tokens gives)
  const int rows = P->B * K, V = P->cfg.vocab, nt = (V + kSampTile - 1) / kSampTile;
  const float inv_t = 1.f / temperature;
  mark(P, ORTHRUS_KIND_SAMPLE, st);
  if (launch(row_stats_kernel, dim3(rows), dim3(kSampThreads), 0, st, (const float*)draft_logits, rows,
             (const float*)nullptr, V, inv_t, P->samp, P->status) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  if (launch(draw_totals_kernel, dim3(rows, (nt + kTotTiles - 1) / kTotTiles), dim3(kTotThreads), 0, st,
             (const float*)draft_logits, V, inv_t, (const float2*)P->samp, P->samp_tot) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  if (launch(draw_select_kernel, dim3(rows), dim3(32), 0, st, (const float*)draft_logits, V, inv_t,
             (const float2*)P->samp, (const float*)P->samp_tot, u_draft, P->draft_ids) != cudaSuccess)
    return ORTHRUS_ERR_CUDA;
  mark(P, ORTHRUS_KIND_END, st);
  s = orthrus_verify_block(plan, pending, P->draft_ids, K, P->ar_ids, verify_logits, stream);
  if (s != ORTHRUS_OK) return s;
  return sampled_consensus(P, pending, P->draft_ids, draft_logits, verify_logits, K, temperature, u_accept, u_final,
                           accept_len, committed, true, st);
}

// ---- single kernels -------------------------------------------------------

size_t orthrus_attention_workspace_bytes(int32_t batch, int32_t n_kv_heads, int32_t group, int32_t Q, int32_t head_dim,
                                         int32_t capacity) {
  if (batch < 1 || n_kv_heads < 1 || group < 1 || Q < 1 || capacity < 1 || (head_dim != 64 && head_dim != 128))
    return 0;
  const int rt = (Q * group + 127) / 128;
  const int ck = attn_chunk_keys(batch, n_kv_heads, rt, capacity);
  const size_t chunks = (capacity + ck - 1) / ck + 1;
  const size_t slots = (size_t)batch * n_kv_heads * rt;
  return align_up(slots * chunks * 128 * head_dim * 4, 256) + align_up(slots * chunks * 128 * 8, 256) +
         align_up(slots * 4, 256);
}

orthrus_status orthrus_attention(const void* q, const void* k_cache, const void* v_cache, const void* k_blk,
                                 const void* v_blk, const int32_t* len, int32_t batch, int32_t n_kv_heads,
                                 int32_t group, int32_t Q, int32_t head_dim, int32_t capacity, int32_t blk_stride,
                                 int32_t mode, void* out, void* workspace, size_t workspace_bytes, int32_t* status,
                                 orthrus_stream stream) {
  if (!q || !k_cache || !v_cache || !len || !out || !workspace || (mode != 0 && mode != 1)) return ORTHRUS_ERR_ARG;
  if (mode == 0 && (!k_blk || !v_blk || blk_stride < Q)) return ORTHRUS_ERR_ARG;
  if (group != 1 && group != 2 && group != 4 && group != 8) return ORTHRUS_ERR_UNSUPPORTED;
  if (Q > 64 && mode == 0) return ORTHRUS_ERR_UNSUPPORTED;
  const size_t need = orthrus_attention_workspace_bytes(batch, n_kv_heads, group, Q, head_dim, capacity);
  if (!need) return ORTHRUS_ERR_ARG;
  if (workspace_bytes < need) return ORTHRUS_ERR_WORKSPACE;
  if (!encode_fn()) return ORTHRUS_ERR_CUDA;
  const int rt = (Q * group + 127) / 128;
  const int ck = attn_chunk_keys(batch, n_kv_heads, rt, capacity);
  const int chunks = (capacity + ck - 1) / ck + 1;
  const size_t slots = (size_t)batch * n_kv_heads * rt;
  char* base = (char*)workspace;
  float* part_o = (float*)base;
  float2* part_ml = (float2*)(base + align_up(slots * chunks * 128 * head_dim * 4, 256));
  int* counter = (int*)(base + align_up(slots * chunks * 128 * head_dim * 4, 256) + align_up(slots * chunks * 128 * 8, 256));
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(counter, 0, slots * 4, st) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkb, tvb;
  const uint64_t z = (uint64_t)batch * n_kv_heads;
  bool ok = map2d(&tq, q, head_dim, z * Q * group, 64, 128, kF16);
  ok = ok && map3d(&tk, k_cache, head_dim, capacity, z, 128, 1, kF16) &&
       map3d(&tv, v_cache, head_dim, capacity, z, 128, 1, kF16);
  if (mode == 0)
    ok = ok && map3d(&tkb, k_blk, head_dim, blk_stride, z, 128, 1, kF16) &&
         map3d(&tvb, v_blk, head_dim, blk_stride, z, 128, 1, kF16);
  else {
    tkb = tk;
    tvb = tv;
  }
  if (!ok) return ORTHRUS_ERR_ARG;
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.B = batch;
  a.Hkv = n_kv_heads;
  a.G = group;
  a.Q = Q;
  a.d = head_dim;
  a.mode = mode;
  a.b0 = 0;
  a.rows = Q * group;
  a.row_tiles = rt;
  a.chunk_keys = ck;
  a.cap = capacity;
  a.z_cache = 0;
  a.z_blk = 0;
  a.max_chunks = (capacity + ck - 1) / ck + (mode == 0 ? 1 : 0);
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
  a.len = len;
  a.out = (__nv_bfloat16*)out;
  a.out_lo = (size_t)batch * Q * n_kv_heads * group * head_dim;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.counter = counter;
  a.status = status;
  return launch_attention(head_dim, tq, tk, tv, tkb, tvb, a, st) == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

size_t orthrus_linear_workspace_bytes(int32_t M, int32_t N, int32_t Kd) {
  if (M < 1 || N < 128 || N % 128 || Kd < 64 || Kd % 64) return 0;
  const size_t tiles = (size_t)((M + 127) / 128) * (N / 128);
  return align_up((size_t)2 * num_sms() * 128 * 128 * 4, 256) + align_up(tiles * 4, 256);
}

orthrus_status orthrus_linear(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t Kd,
                              void* workspace, size_t workspace_bytes, int32_t* status, orthrus_stream stream) {
  if (!X || !W || !Y || !workspace) return ORTHRUS_ERR_ARG;
  const size_t need = orthrus_linear_workspace_bytes(M, N, Kd);
  if (!need) return ORTHRUS_ERR_UNSUPPORTED;
  if (workspace_bytes < need) return ORTHRUS_ERR_WORKSPACE;
  if (!encode_fn()) return ORTHRUS_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)workspace;
  const size_t part_bytes = align_up((size_t)2 * num_sms() * 128 * 128 * 4, 256);
  int* cnt = (int*)(base + part_bytes);
  const size_t tiles = (size_t)((M + 127) / 128) * (N / 128);
  if (cudaMemsetAsync(cnt, 0, tiles * 4, st) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  CUtensorMap tw, tx;
  if (!map2d(&tw, W, Kd, N, 64, 128) || !map2d(&tx, X, Kd, M, 64, 16 * (mt_index(M) + 1))) return ORTHRUS_ERR_ARG;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.partial = (float*)base;
  a.tile_counter = cnt;
  a.status = status;
  a.out_f32 = Y;
  a.ld_out = N;
  return launch_gemm<EPI_STORE>(tw, tx, a, N, Kd, M, st) == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// orthrus_linear_noalloc: orthrus_linear with its scratch in a static device array
// ---------------------------------------------------------------------------
// Scratch of the stream-K GEMM: partial sums of split weight tiles (one 128 x 128
// fp32 slot pair per CTA) and the tiles' arrival counters. The grid is capped at
// kNoAllocCtas CTAs so the partial slots fit; the counters cover kNoAllocTiles
// tiles. Every GPU that loads the library holds this array until the process exits.
namespace {
constexpr int kNoAllocCtas = 32;
constexpr size_t kNoAllocPartialBytes = (size_t)2 * kNoAllocCtas * 128 * 128 * 4;  // 4 MiB
constexpr int kNoAllocTiles = 16384;
constexpr size_t kNoAllocBytes = kNoAllocPartialBytes + (size_t)kNoAllocTiles * 4;  // 4 MiB + 64 KiB
}  // namespace

static __device__ __align__(256) unsigned char g_linear_scratch[kNoAllocBytes];

namespace {
// Device address of g_linear_scratch on the current device, looked up once per
// device (host code cannot use the symbol itself as a device address).
void* linear_scratch_address() {
  static std::mutex mu;
  static void* addr[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || !p) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

template <int EPI>
cudaError_t launch_gemm_capped(const CUtensorMap& tmW, const CUtensorMap& tmX, GemmArgs a, int N, int Kd, int M,
                               int max_ctas, cudaStream_t st) {
  a.N = N;
  a.Kd = Kd;
  a.M = M;
  a.m_tiles = (M + 127) / 128;
  a.Mt = a.m_tiles > 1 ? 128 : round_up(std::max(M, 1), 16);
  a.mt_alloc = std::max(32, next_pow2(a.Mt));
  a.n_tiles = N / 128;
  a.k_chunks = Kd / 64;
  a.total_units = (long long)a.m_tiles * a.n_tiles * a.k_chunks;
  const int G = (int)std::min<long long>(std::min(num_sms(), max_ctas), a.total_units);
  a.planes = 1;  // the caller's X is one bf16 matrix
  const size_t fixed = gemm_smem_bytes(a.Mt, 0, 1);
  const size_t stage = 16384 + (size_t)a.Mt * 128;
  a.stages = (int)std::min<size_t>(12, (kSmemLimit - fixed) / stage);
  const size_t smem = gemm_smem_bytes(a.Mt, a.stages, 1);
  if (!ensure_smem_attr(gemm_kernel<EPI>, kSmemLimit)) return cudaErrorInvalidValue;
  return launch(gemm_kernel<EPI>, dim3(G), dim3(kGemmThreads), smem, st, tmW, tmX, a);
}
}  // namespace

extern "C" orthrus_status orthrus_linear_noalloc(const void* X, const void* W, float* Y, int32_t M, int32_t N,
                                                 int32_t Kd, int32_t* status, orthrus_stream stream) {
  if (!X || !W || !Y) return ORTHRUS_ERR_ARG;
  if (M < 1 || N < 128 || N % 128 || Kd < 64 || Kd % 64) return ORTHRUS_ERR_UNSUPPORTED;
  const long long tiles = (long long)((M + 127) / 128) * (N / 128);
  if (tiles > kNoAllocTiles) return ORTHRUS_ERR_WORKSPACE;  // beyond the static scratch
  if (!encode_fn()) return ORTHRUS_ERR_CUDA;
  char* base = (char*)linear_scratch_address();
  if (!base) return ORTHRUS_ERR_CUDA;
  int* cnt = (int*)(base + kNoAllocPartialBytes);
  cudaStream_t st = (cudaStream_t)stream;
  // the array keeps the previous call's contents: the arrival counters must start at zero
  if (cudaMemsetAsync(cnt, 0, (size_t)tiles * 4, st) != cudaSuccess) return ORTHRUS_ERR_CUDA;
  CUtensorMap tw, tx;
  if (!map2d(&tw, W, Kd, N, 64, 128) || !map2d(&tx, X, Kd, M, 64, 16 * (mt_index(M) + 1))) return ORTHRUS_ERR_ARG;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.partial = (float*)base;
  a.tile_counter = cnt;
  a.status = status;
  a.out_f32 = Y;
  a.ld_out = N;
  return launch_gemm_capped<EPI_STORE>(tw, tx, a, N, Kd, M, kNoAllocCtas, st) == cudaSuccess ? ORTHRUS_OK
                                                                                            : ORTHRUS_ERR_CUDA;
}
