// Persistent forward kernel: one launch runs a whole draft-view or verify-view
// forward of the Orthrus decode step (embedding, every layer's q/k/v
// projection, block attention, output projection, SwiGLU MLP, final norm, LM
// head and argmax) for a block whose token rows fit two ring stages (at most 96 at
// head dim 128), and the verify launch also runs the greedy consensus and KV commit
// at its end.
//
// Why one kernel: at decode sizes every projection is a weight stream of 5-30
// microseconds, so separate launches pay a start-up and a split-K tail per
// projection (hundreds per step) that are as long as the stream itself. Here
// one CTA per SM (cooperative launch, all CTAs co-resident) walks the same list
// of phases; the phases are ordered by device-wide counters instead of kernel
// boundaries, and the TMA producer keeps streaming the next phase's weight
// tiles into its shared-memory ring while the current phase finishes, so the
// weight stream does not stop at phase boundaries.
//
// Phases of one forward (phase p depends on the previous active phase only):
//   EMBED         h = E[ids], xg = split(h * gamma_attn[0]), per-row sums of squares
//   per layer:
//     QKV         [xg] W_qkv^T, * rstd, per-head q/k RMSNorm, RoPE; q -> qbuf, K/V ->
//                 cache slots len+i (verify) or the draft block scratch (draft)
//     ATTN        block attention over (sequence, kv head, 128-row tile, key chunk) units
//     COMBINE     merge of the key-chunk partials (only when some slot has several chunks)
//     O           h += attn W_o^T; xg = split(h * gamma_mlp); sums of squares
//     GU          act = silu(rstd * xg W_g^T) * (rstd * xg W_u^T)
//     DOWN        h += act W_down^T; xg = split(h * gamma_next); sums of squares
//   LM            logits = rstd * xg W_lm^T; running argmax per row
// RMSNorm is folded into its neighbours: RMSNorm(h) W^T = diag(rstd) (h*gamma) W^T,
// so the residual epilogue writes split(h * gamma) and 128-column partial sums of
// h^2, and the consumer multiplies its accumulator rows by rstd, computed from the
// partial sums in a fixed order (deterministic).
//
// Operand precision. Over 36 layers every bf16 rounding of an activation adds to the
// logits' error, so the operands carry more bits than bf16:
//   - an activation that feeds a layer projection (xg, the attention output, the SwiGLU
//     output) is written as two bf16 planes, hi = bf16(x) and lo = bf16(x - hi); every
//     weight chunk is multiplied with both in one MMA (N = 2 Mt: the hi rows, then the lo
//     rows; the two fp32 accumulators sit side by side in TMEM and the epilogue adds
//     them), so the projection sees x to about 2^-17 relative. The LM head reads the hi
//     plane only;
//   - attention runs on fp16 operands: q and the softmax weights P (11 significant bits),
//     and K/V, bf16 values held in the fp16 encoding.
//
// Warp roles (224 threads): warp 0 = TMA producer of weight tiles, warp 6 = TMA
// producer of activation tiles (the loads that wait for the previous phase), warp
// 1 = tcgen05.mma issuer, warps 2-5 = epilogue (TMEM -> registers -> fused
// epilogue), attention softmax, embedding and chunk merge. Two issuing threads
// matter: one thread issuing 8 KB copies streams about 4 TB/s, two reach the
// HBM rate. Ring stage = a 32 KB weight box (128 rows x two 64-wide k chunks) + an
// activation box of Mt rows x two k chunks x two planes; in attention phases a stage
// holds one 64-key tile's K, V and P tile instead.
#pragma once
#include "gemm.cuh"

namespace orthrus {

// tensor-map indices: per layer, then global
// The persistent kernel reads every projection through a 3-D view (64 columns, rows,
// k chunk of 64) with strides (row, 128 bytes): one 32 KB box brings two consecutive
// 64-wide k chunks of 128 rows (256 contiguous bytes per row), which streams about
// 10% faster than two 16 KB boxes. M_WGU4 adds the gate/up half as a 4th dimension,
// so a box holds, per k chunk, 64 gate rows and the 64 matching up rows.
// The per-op kernels use the 2-D maps (M_WQKV .. M_WDO).
enum {
  M_WQKV = 0,
  M_WO,
  M_WGU,
  M_WDOWN,
  M_WDQKV,
  M_WDO,
  M_WQKV3,
  M_WO3,
  M_WDOWN3,
  M_WDQKV3,
  M_WDO3,
  M_WGU4,
  M_PER_LAYER
};
// activation maps exist for every token-tile height Mt = 16, 32, ..., 128 (index Mt/16 - 1)
enum {
  G_LM = 0,
  G_Q,
  G_KC,
  G_VC,
  G_KB,
  G_VB,
  G_KC64,
  G_VC64,
  G_KB64,
  G_VB64,
  G_XN,                 // normalised input, hi plane only (the LM head's operand)
  G_XNP = G_XN + 8,     // normalised input, both planes: (64 columns, rows, plane)
  G_ATTN = G_XNP + 8,   // attention output, both planes
  G_ACT = G_ATTN + 8,   // SwiGLU output, both planes
  G_LM3 = G_ACT + 8,    // k-pair views of the LM head and of the activations (persistent kernel)
  G_XN3,                // hi plane: (64 columns, rows, k chunk)
  G_XN4 = G_XN3 + 8,    // both planes: (64 columns, rows, k chunk, plane)
  G_ATTN4 = G_XN4 + 8,
  G_ACT4 = G_ATTN4 + 8,
  G_COUNT = G_ACT4 + 8
};

enum PhaseKind : int { PH_EMBED = 0, PH_QKV, PH_ATTN, PH_COMBINE, PH_O, PH_GU, PH_DOWN, PH_LM };
constexpr int kPhasesPerLayer = 6;  // QKV, ATTN, COMBINE, O, GU, DOWN
constexpr int kFwdThreads = 224;
constexpr int kMaxStages = 16;
constexpr int kMaxSlots = 256;        // attention (sequence, kv head, row tile) slots per launch
constexpr int kMaxChunks = 34;        // key chunks per slot (32 cache chunks + draft block + slack)
constexpr int kCombineRows = 16;      // rows per merge unit
constexpr int kScratchBytes = 19584;  // epilogue staging (36 x 132 fp32 + per-quarter sums)
constexpr int kMaxGrid = 256;         // CTAs (one per SM) the unit-range table covers
constexpr float kRescaleLog2 = 8.f;   // attention: largest log2 step of a score over the exponent offset

struct LayerNorms {  // device-resident per-layer gains (fp32)
  const float *attn_norm, *mlp_norm, *q_norm, *k_norm, *wd_q_norm, *wd_k_norm;
};

struct FwdArgs {
  const CUtensorMap* maps;   // device copy: [L][M_PER_LAYER] then [G_COUNT]
  const LayerNorms* norms;   // device [L]
  int L, D, H, Hkv, d, F, V, G, qk_norm, mask_id;
  float eps, scale_log2;
  double theta;
  int view;                  // VIEW_DRAFT / VIEW_VERIFY
  int nb, Q, M, Mt, mt_idx, stages, cap, max_block, batch;
  int lookahead;             // weight tiles the weight producer loads ahead of a phase's input dependency
  int poll_ns;               // sleep between polls of a phase counter
  int ck;                    // keys per attention chunk: fixed per plan (multiple of 64, >= capacity / 32),
                             // so a row's softmax runs over the same absolute key chunks whatever
                             // the block size: verify rows equal the plain AR rows bit for bit
  const int* pending;        // [nb]
  const int* draft_ids;      // verify: [nb][Q-1]; draft: nullable [nb][Q], the previous drafts
  int* len;                  // [batch] (read; the fused accept advances it)
  const __nv_bfloat16* embed;
  const float* final_norm;
  __half *kc, *vc, *blk_k, *blk_v;  // bf16 values in the fp16 encoding
  float* h;                  // [rows][D]
  __nv_bfloat16* xg;         // [2][rows][D]: hi plane, then lo plane at + xg_lo
  __half* qbuf;              // [nb][Hkv][Q*G][d]
  __nv_bfloat16* attn;       // [2][rows][H*d] (lo plane at + attn_lo)
  __nv_bfloat16* act;        // [2][rows][F] (lo plane at + act_lo)
  size_t xg_lo, attn_lo, act_lo;  // element offsets of the lo planes
  float2* rope;              // [rows][d/2]
  float* ss;                 // [D/128][ss_ld] partial sums of squares
  int ss_ld;
  unsigned long long* amax;  // [rows]
  int* out_ids;              // [M] argmax of every row
  float* logits;             // nullable [M][V]
  float* partial;            // [2 * grid][128][Mt] split-tile partial sums
  int* tile_cnt;             // [max tiles] split-tile arrival counters (self-resetting)
  int* phase_cnt;            // [2 + 6L] completion counters (reset by the last CTA)
  int* exit_cnt;
  float* att_o;              // [kMaxSlots][kMaxChunks][128][d]
  float2* att_ml;            // [kMaxSlots][kMaxChunks][128]
  int* status;
  int* diag;                 // [16] where the first timed-out wait gave up (nullable)
  unsigned long long* tl;    // nullable [grid][phases][8] event times (profiling)
  // greedy consensus fused into the verify launch
  int accept, K;
  int* pending_out;          // [nb]
  int* accept_len;           // [nb]
  int* committed;            // [nb][K+1]
};

// Records the first wait that ran out of time: site, phase, ring position and
// two site-specific values (diag[0] = 1 once written).
__device__ __noinline__ void fwd_diag(const FwdArgs& a, int code, int site, int p, int it, int x0 = 0, int x1 = 0,
                                int x2 = 0) {
  if (code != -1 || !a.diag) return;
  if (atomicCAS(a.diag, 0, 1) != 0) return;
  a.diag[1] = blockIdx.x;
  a.diag[2] = threadIdx.x;
  a.diag[3] = site;
  a.diag[4] = p;
  a.diag[5] = it;
  a.diag[6] = x0;
  a.diag[7] = x1;
  a.diag[8] = x2;
  __threadfence();
}

// Phase timeline events (globaltimer, ns), per CTA and phase:
//   0/1 weight producer first/last load issued, 2/3 activation producer dependency
//   met / last load issued, 4/5 first MMA / last MMA commit, 6/7 epilogue
//   dependency met / phase finished.
//   8..13 (last epilogue segment of a projection phase): accumulator ready, partial
//   stored, arrival counted, partials loaded, epilogue done, completion signalled.
enum { TL_W0 = 0, TL_W1, TL_X0, TL_X1, TL_M0, TL_M1, TL_E0, TL_E1, TL_S_ACC, TL_S_PART, TL_S_CNT, TL_S_LOAD,
       TL_S_EPI, TL_S_SIG, TL_R0, TL_R1, TL_EVENTS };
// The marks exist only in the profiling instantiation of the kernel (TL = true):
// their address arithmetic and stores change register allocation around them.
template <bool TL>
__device__ __forceinline__ void tl_mark(const FwdArgs& a, int n_ph, int p, int ev) {
  if constexpr (!TL) return;
  if (a.tl) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)::"memory");  // not moved across memory operations
    a.tl[((size_t)blockIdx.x * n_ph + p) * TL_EVENTS + ev] = t;
  }
}

__host__ __device__ inline int fwd_n_phases(int L) { return 2 + kPhasesPerLayer * L; }
__host__ __device__ inline int fwd_phase_kind(int p, int L) {
  if (p == 0) return PH_EMBED;
  if (p == 1 + kPhasesPerLayer * L) return PH_LM;
  return PH_QKV + (p - 1) % kPhasesPerLayer;
}
__host__ __device__ inline int fwd_phase_layer(int p) { return (p - 1) / kPhasesPerLayer; }

// Shared memory outside the ring: the attention Q tile (128 rows x d, resident for
// a whole attention unit, so it cannot live in the ring), the epilogue staging, small
// per-CTA tables and the barriers. (Attention's P tiles live in the ring stages.)
__host__ inline size_t fwd_fixed_smem(int d) {
  return 1024 /*align*/ + (size_t)128 * d * 2 /*Q*/ + kScratchBytes + 144 * 8 /*red*/ + 128 * 4 /*rstd*/ +
         128 * 4 /*lens*/ + (kMaxSlots + 1) * 4 /*slot prefix*/ + 64 * 8 /*barriers*/ + 64 * 4 /*misc*/ +
         kMaxGrid * 4 /*unit-range starts*/;
}
// ring stage: 32 KB weight box (128 rows x two k chunks) + activation box (Mt rows x two k
// chunks x two planes; the LM head reads the hi plane only)
// In attention phases a stage holds one 64-key tile: K, V (64 x d fp16 each) and its P tile
// (128 rows x 64 keys fp16).
__host__ __device__ inline uint32_t fwd_stage_bytes(int Mt, int d) {
  const uint32_t proj = 32768u + (uint32_t)Mt * 512u, att = 2u * 128u * (uint32_t)d + 16384u;
  return proj > att ? proj : att;
}

// Shared state every role derives identically at kernel start.
struct FwdGeom {
  int rows_per_slot;  // Q * G
  int rt;             // row tiles per (sequence, kv head)
  int slots;          // nb * Hkv * rt
  int CK;             // keys per chunk (multiple of 64)
  int att_units;      // total attention units
  int comb_units;     // total merge units (0 when no slot has more than one chunk)
};

// GEMM phase description
struct GemmPhase {
  int epi;            // EPI_QKV / EPI_RESID / EPI_SWIGLU / EPI_ARGMAX
  int n_tiles, k_chunks;  // k_chunks: 128-wide k units per tile (each a pair of 64-wide chunks)
  long long units;
  const CUtensorMap* mw;
  const CUtensorMap* mx;
  int gu;             // SwiGLU tile layout (64 gate + 64 up rows)
  int planes;         // activation planes: 2 (hi + lo) for the layer projections, 1 for the LM head
};

__device__ inline GemmPhase gemm_phase(const FwdArgs& a, int kind, int l) {
  GemmPhase g;
  const CUtensorMap* lm = a.maps + (size_t)l * M_PER_LAYER;
  const CUtensorMap* gm = a.maps + (size_t)a.L * M_PER_LAYER;
  const bool draft = a.view == VIEW_DRAFT;
  g.gu = 0;
  g.planes = 2;
  if (kind == PH_QKV) {
    g.epi = EPI_QKV;
    g.n_tiles = (a.H + 2 * a.Hkv) * a.d / 128;
    g.k_chunks = a.D / 128;
    g.mw = lm + (draft ? M_WDQKV3 : M_WQKV3);
    g.mx = gm + G_XN4 + a.mt_idx;
  } else if (kind == PH_O) {
    g.epi = EPI_RESID;
    g.n_tiles = a.D / 128;
    g.k_chunks = a.H * a.d / 128;
    g.mw = lm + (draft ? M_WDO3 : M_WO3);
    g.mx = gm + G_ATTN4 + a.mt_idx;
  } else if (kind == PH_GU) {
    g.epi = EPI_SWIGLU;
    g.n_tiles = a.F / 64;
    g.k_chunks = a.D / 128;
    g.mw = lm + M_WGU4;
    g.mx = gm + G_XN4 + a.mt_idx;
    g.gu = 1;
  } else if (kind == PH_DOWN) {
    g.epi = EPI_RESID;
    g.n_tiles = a.D / 128;
    g.k_chunks = a.F / 128;
    g.mw = lm + M_WDOWN3;
    g.mx = gm + G_ACT4 + a.mt_idx;
  } else {  // PH_LM
    g.epi = EPI_ARGMAX;
    g.n_tiles = a.V / 128;
    g.k_chunks = a.D / 128;
    g.mw = gm + G_LM3;
    g.mx = gm + G_XN3 + a.mt_idx;
    g.planes = 1;
  }
  g.units = (long long)g.n_tiles * g.k_chunks;
  return g;
}

__device__ inline bool is_gemm_kind(int k) {
  return k == PH_QKV || k == PH_O || k == PH_GU || k == PH_DOWN || k == PH_LM;
}

// completion count of a phase
__device__ inline int phase_target(const FwdArgs& a, const FwdGeom& g, int p) {
  const int kind = fwd_phase_kind(p, a.L);
  if (kind == PH_EMBED) return a.M;
  if (kind == PH_ATTN) return g.att_units;
  if (kind == PH_COMBINE) return g.comb_units;
  return gemm_phase(a, kind, 0).n_tiles;
}

__device__ inline bool phase_active(const FwdGeom& g, int kind) { return kind != PH_COMBINE || g.comb_units > 0; }

// the phase whose completion phase p waits for (the previous active phase)
__device__ inline int phase_dep(const FwdArgs& a, const FwdGeom& g, int p) {
  int q = p - 1;
  if (q >= 1 && !phase_active(g, fwd_phase_kind(q, a.L))) --q;
  return q;
}

// ---- attention geometry ------------------------------------------------------
// slot s = (bb * Hkv + kvh) * rt + r
__device__ inline int slot_visible_keys(const FwdArgs& a, const FwdGeom& g, const int* lens, int s) {
  const int r = s % g.rt;
  const int bb = s / (g.rt * a.Hkv);
  const int n = min(lens[bb], a.cap);
  if (a.view == VIEW_DRAFT) return n;  // cache keys; the block is one extra chunk
  const int row_hi = min(g.rows_per_slot, (r + 1) * 128);
  const int i_max = (row_hi - 1) / a.G;
  return min(n + i_max + 1, a.cap);
}

__device__ inline int slot_chunks(const FwdArgs& a, const FwdGeom& g, const int* lens, int s) {
  const int vis = slot_visible_keys(a, g, lens, s);
  const int c = (vis + g.CK - 1) / g.CK;
  return a.view == VIEW_DRAFT ? c + 1 : max(1, c);
}

}  // namespace orthrus

namespace orthrus {

struct AttUnit {
  int slot, chunk, n_chunks, bb, kvh, r, blk, key_lo, key_hi, n, tiles;
};

// attention unit u -> (slot, key chunk, key range); slot_pre = prefix sums of chunks per slot
__device__ inline AttUnit att_unit(const FwdArgs& a, const FwdGeom& g, const int* lens, const int* slot_pre, int u) {
  int lo = 0, hi = g.slots - 1;  // largest s with slot_pre[s] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (slot_pre[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  AttUnit t;
  t.slot = lo;
  t.chunk = u - slot_pre[lo];
  t.n_chunks = slot_pre[lo + 1] - slot_pre[lo];
  t.r = lo % g.rt;
  t.kvh = (lo / g.rt) % a.Hkv;
  t.bb = lo / (g.rt * a.Hkv);
  t.n = min(lens[t.bb], a.cap);
  const int vis = slot_visible_keys(a, g, lens, lo);
  if (a.view == VIEW_DRAFT && t.chunk == t.n_chunks - 1) {
    t.blk = 1;
    t.key_lo = 0;
    t.key_hi = a.Q;
  } else {
    t.blk = 0;
    t.key_lo = t.chunk * g.CK;
    t.key_hi = min(vis, t.key_lo + g.CK);
  }
  t.tiles = max(1, (t.key_hi - t.key_lo + 63) / 64);
  return t;
}

// The epilogues below stage the 128 x 32 accumulator group in shared memory
// (thread = tile row `row`, v[j] = token j), then re-read it with one thread per
// (token row, quarter of the tile): lane = token row, warp = quarter for the
// residual and SwiGLU epilogues (conflict-free 16-byte reads: the staging row
// stride shifts each row by four banks), four adjacent lanes per token row for
// the q/k/v epilogue (so a head's sum of squares is two shuffles). Every thread
// then runs the same short code and stores 16-byte vectors.

// Scratch layout of the epilogues (floats): the 32-row staging tile [32][kEpiStride],
// 128 per-quarter sums, then the second group's staging [4][kEpiStride] and its 16
// per-quarter sums. The second group carries token rows [m0+32, m0+32+n2), n2 <= 4:
// the 33rd row of a K = 32 verify block goes through the same call as the first 32.
constexpr int kEpiQsum = 32 * kEpiStride;
constexpr int kEpi2 = kEpiQsum + 128;
constexpr int kEpi2Qsum = kEpi2 + 4 * kEpiStride;
constexpr int kEpiFloats = kEpi2Qsum + 16;
static_assert(kEpiFloats * 4 <= kScratchBytes, "epilogue scratch");

// second-group token count of a call on rows [m0, ...): rows past m0+32 when the block ends
// within 4 of them (else the caller runs a separate call per 32 rows)
__device__ __forceinline__ int epi_group2(int m0, int m_valid) {
  const int n = m_valid - m0 - 32;
  return n > 0 && n <= 4 ? n : 0;
}

// one (token row, 32-column quarter) of the residual epilogue: h row -> global, xg = bf16(h * gamma)
// -> global; returns the quarter's sum of squares
__device__ __forceinline__ float resid_quarter(const FwdArgs& a, const float* src, int m, int nt, int qq, bool store,
                                               const float* gam_t) {
  const int D = a.D;
  float y[32];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 f4 = *reinterpret_cast<const float4*>(src + 4 * c);
    y[4 * c] = f4.x;
    y[4 * c + 1] = f4.y;
    y[4 * c + 2] = f4.z;
    y[4 * c + 3] = f4.w;
  }
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    s0 += y[i] * y[i];
    s1 += y[i + 1] * y[i + 1];
    s2 += y[i + 2] * y[i + 2];
    s3 += y[i + 3] * y[i + 3];
  }
  if (store) {
    float4* hp = reinterpret_cast<float4*>(a.h + (size_t)m * D + nt * 128 + qq * 32);
#pragma unroll
    for (int c = 0; c < 8; ++c) hp[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
    const float4* gq = reinterpret_cast<const float4*>(gam_t + qq * 32);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 g4 = gq[c];
      y[4 * c] *= g4.x, y[4 * c + 1] *= g4.y, y[4 * c + 2] *= g4.z, y[4 * c + 3] *= g4.w;
    }
    __nv_bfloat16* xp = a.xg + (size_t)m * D + nt * 128 + qq * 32;
    st_split_x16(xp, xp + a.xg_lo, y);
    st_split_x16(xp + 16, xp + a.xg_lo + 16, y + 16);
  }
  return (s0 + s1) + (s2 + s3);
}

// Residual epilogue of the O and down projections on token rows [m0, m0+32) (+ the second
// group v2) of one 128-column tile: h += v; xg = bf16(h * gamma_next); sum of h^2 over the
// tile's 128 columns per row -> ss[nt][m]. With h_in_v the old h is already part of v (added
// by the contributor that holds the tile's last k-chunk, early in its range, so no h load
// sits on the path). gam_t: the next norm's gains of this tile's 128 columns.
__device__ __forceinline__ void fwd_resid_epilogue(const FwdArgs& a, const float* v, const float* v2, int row, int m0,
                                                   int nt, int m_valid, const float* gam_t, float* epi, bool h_in_v) {
  const int D = a.D;
  const int n2 = v2 ? epi_group2(m0, m_valid) : 0;
  if (h_in_v) {
#pragma unroll
    for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < n2) epi[kEpi2 + k * kEpiStride + row] = v2[k];
  } else {
    float hv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      hv[j] = m0 + j < m_valid ? __ldcg(a.h + (size_t)(m0 + j) * D + nt * 128 + row) : 0.f;
    float hv2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) hv2[k] = k < n2 ? __ldcg(a.h + (size_t)(m0 + 32 + k) * D + nt * 128 + row) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j] + hv[j];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < n2) epi[kEpi2 + k * kEpiStride + row] = v2[k] + hv2[k];
  }
  named_bar_sync(1, 128);
  const int t = threadIdx.x - 64, j = t & 31, qq = t >> 5;
  epi[kEpiQsum + qq * 32 + j] =
      resid_quarter(a, epi + j * kEpiStride + qq * 32, m0 + j, nt, qq, m0 + j < m_valid, gam_t);
  if (t < 4 * n2) {  // second group: thread = (row k, quarter q2)
    const int k = t >> 2, q2 = t & 3;
    epi[kEpi2Qsum + q2 * 4 + k] = resid_quarter(a, epi + kEpi2 + k * kEpiStride + q2 * 32, m0 + 32 + k, nt, q2, true, gam_t);
  }
  named_bar_sync(1, 128);
  if (t < 32 && m0 + t < m_valid) {
    const float* q = epi + kEpiQsum;
    a.ss[(size_t)nt * a.ss_ld + m0 + t] = ((q[t] + q[32 + t]) + q[64 + t]) + q[96 + t];
  } else if (t >= 32 && t < 32 + n2) {
    const int k = t - 32;
    const float* q = epi + kEpi2Qsum;
    a.ss[(size_t)nt * a.ss_ld + m0 + 32 + k] = ((q[k] + q[4 + k]) + q[8 + k]) + q[12 + k];
  }
}

// Per-phase state of the q/k/v projection epilogue: destination of the block's
// K/V, the q/k RMSNorm gains (gains[0, d) for q, gains[d, 2d) for k) and the RoPE
// factors of token rows [0, rope_rows) (both in shared memory; rows past
// rope_rows read the global table).
struct QkvCtx {
  __half *kdst, *vdst;
  int kv_stride;
  const float* gains;
  const float2* rope;
  int rope_rows;
};

// one (token row m, quarter qq) of the q/k/v epilogue; src = the row's staged 128 columns.
// Every lane of the warp runs it (the head's sum of squares is two shuffles); lanes with
// valid == false store nothing.
template <int D_HEAD>
__device__ __forceinline__ void qkv_item(const FwdArgs& a, const QkvCtx& q, const float* src_row, int m, int nt,
                                         int qq, bool valid, const int* lens_s) {
  constexpr int d = D_HEAD, half = d / 2, TPH = d / 32;
  const int hl = qq / TPH, e0 = 16 * (qq % TPH);
  const int hh = (nt * 128) / d + hl;  // head index in the fused q|k|v rows
  const int kind = hh < a.H ? 0 : (hh < a.H + a.Hkv ? 1 : 2);
  const float* src = src_row + hl * d;
  float x1[16], x2[16];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 f1 = *reinterpret_cast<const float4*>(src + e0 + 4 * c);
    const float4 f2 = *reinterpret_cast<const float4*>(src + half + e0 + 4 * c);
    x1[4 * c] = f1.x, x1[4 * c + 1] = f1.y, x1[4 * c + 2] = f1.z, x1[4 * c + 3] = f1.w;
    x2[4 * c] = f2.x, x2[4 * c + 1] = f2.y, x2[4 * c + 2] = f2.z, x2[4 * c + 3] = f2.w;
  }
  // sum of squares over the head: own 32 elements, then the other TPH-1 threads
  // (adjacent lanes); every lane shuffles, whatever its head's kind
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    s0 += x1[i] * x1[i];
    s1 += x1[i + 1] * x1[i + 1];
    s2 += x2[i] * x2[i];
    s3 += x2[i + 1] * x2[i + 1];
  }
  float ss = (s0 + s1) + (s2 + s3);
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  if (TPH == 4) ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  if (kind < 2) {
    if (a.qk_norm) {
      const float rr = rsqrtf(ss * (1.0f / d) + a.eps);
      const float4* g1 = reinterpret_cast<const float4*>(q.gains + (kind == 0 ? 0 : d) + e0);
      const float4* g2 = g1 + half / 4;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 a1 = g1[c], a2 = g2[c];
        x1[4 * c] *= rr * a1.x, x1[4 * c + 1] *= rr * a1.y, x1[4 * c + 2] *= rr * a1.z, x1[4 * c + 3] *= rr * a1.w;
        x2[4 * c] *= rr * a2.x, x2[4 * c + 1] *= rr * a2.y, x2[4 * c + 2] *= rr * a2.z, x2[4 * c + 3] *= rr * a2.w;
      }
    }
    // element e pairs with e + d/2
    auto rot = [&](int i, float c, float sn) {
      const float y1 = x1[i] * c - x2[i] * sn;
      const float y2 = x2[i] * c + x1[i] * sn;
      x1[i] = y1;
      x2[i] = y2;
    };
    if (m < q.rope_rows) {
      // staged rows: 16-byte chunk c of segment s sits at chunk s*8 + ((c + 2s + (m & 1)) & 7) of the row
      // (the eight lanes of one shared-memory wavefront then hit eight different bank groups)
      const int sg = e0 / 16;
      const float4* rp = reinterpret_cast<const float4*>(q.rope + (size_t)m * half) + sg * 8;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 f = rp[(c + 2 * sg + (m & 1)) & 7];
        rot(2 * c, f.x, f.y);
        rot(2 * c + 1, f.z, f.w);
      }
    } else if (valid) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 f = a.rope[(size_t)m * half + e0 + i];
        rot(i, f.x, f.y);
      }
    }
  }
  if (valid) {
    const int bb = a.nb == 1 ? 0 : m / a.Q, i = m - bb * a.Q;  // (runtime divides cost ~100 cycles each)
    __half* dst = nullptr;
    if (kind == 0) {
      const int G = a.G;
      const int kvh = (G & (G - 1)) == 0 ? hh >> (31 - __clz(G)) : hh / G, g = hh - kvh * G;
      dst = a.qbuf + ((size_t)(bb * a.Hkv + kvh) * (a.Q * G) + i * G + g) * d;
    } else {
      const int kvh = hh - a.H - (kind == 2 ? a.Hkv : 0);
      const int slot = a.view == VIEW_DRAFT ? i : lens_s[bb] + i;
      if (slot >= 0 && slot < q.kv_stride)
        dst = (kind == 1 ? q.kdst : q.vdst) + ((size_t)(bb * a.Hkv + kvh) * q.kv_stride + slot) * d;
#pragma unroll
      for (int e = 0; e < 16; ++e) {  // K and V keep bf16 values (the cache precision)
        x1[e] = kv_value(x1[e]);
        x2[e] = kv_value(x2[e]);
      }
    }
    if (dst) {
      st_f16x16(dst + e0, x1);
      st_f16x16(dst + half + e0, x2);
    }
  }
}

// q/k/v epilogue on token rows [m0, m0+32) (+ the second group v2) of one 128-row tile (one
// head at d = 128, two at d = 64): per-head RMSNorm of q and k, rotate-half RoPE at the row's
// absolute position, bf16 store of q (qbuf) and of k, v (cache slot len+i in the verify view,
// block-scratch row i in the draft view). Thread = (token row j, quarter qq): d/32 threads per
// head, each holding elements [16s, 16s+16) and their RoPE partners [d/2 + 16s, d/2 + 16s + 16).
// The second group's (row, quarter) items run on the first warp.
template <int D_HEAD>
__device__ __forceinline__ void fwd_qkv_epilogue(const FwdArgs& a, const QkvCtx& q, const float* v, const float* v2,
                                                 int row, int m0, int nt, int m_valid, float* epi, const int* lens_s) {
  const int n2 = v2 ? epi_group2(m0, m_valid) : 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < n2) epi[kEpi2 + k * kEpiStride + row] = v2[k];
  named_bar_sync(1, 128);
  const int t = threadIdx.x - 64, j = t >> 2, qq = t & 3;
  qkv_item<D_HEAD>(a, q, epi + j * kEpiStride, m0 + j, nt, qq, m0 + j < m_valid, lens_s);
  if (n2 > 0 && t < 32) {  // warp-uniform
    const int k = min(j, 3);
    qkv_item<D_HEAD>(a, q, epi + kEpi2 + k * kEpiStride, m0 + 32 + k, nt, qq, j < n2, lens_s);
  }
  named_bar_sync(1, 128);
}

// SwiGLU epilogue of the gate/up projection on 32 token rows [m0, m0+32) of one
// tile: rows 0..63 are the gate rows of features nt*64.., rows 64..127 the matching
// up rows; act = silu(gate) * up in bf16. Thread = (token row, 16 features).
// one (token row, 16 features) of the SwiGLU epilogue; src = the row's staged columns
__device__ __forceinline__ void swiglu_item(const FwdArgs& a, const float* src, int m, int nt, int qq) {
  float y[16];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 g4 = *reinterpret_cast<const float4*>(src + 4 * c);
    const float4 u4 = *reinterpret_cast<const float4*>(src + 64 + 4 * c);
    const float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)  // fast reciprocal: an IEEE divide branches per element
      y[4 * c + i] = __fdividef(g[i], 1.0f + __expf(-g[i])) * u[i];
  }
  __nv_bfloat16* dst = a.act + (size_t)m * a.F + nt * 64 + 16 * qq;
  st_split_x16(dst, dst + a.act_lo, y);
}

__device__ __forceinline__ void fwd_swiglu_epilogue(const FwdArgs& a, const float* v, const float* v2, int row, int m0,
                                                    int nt, int m_valid, float* epi) {
  const int n2 = v2 ? epi_group2(m0, m_valid) : 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < n2) epi[kEpi2 + k * kEpiStride + row] = v2[k];
  named_bar_sync(1, 128);
  const int t = threadIdx.x - 64, j = t & 31, qq = t >> 5;
  if (m0 + j < m_valid) swiglu_item(a, epi + j * kEpiStride + 16 * qq, m0 + j, nt, qq);
  if (t < 4 * n2) swiglu_item(a, epi + kEpi2 + (t >> 2) * kEpiStride + 16 * (t & 3), m0 + 32 + (t >> 2), nt, t & 3);
  named_bar_sync(1, 128);
}

// Greedy head of the LM projection on 32 token rows [m0, m0+32) of one 128-row
// vocabulary tile: optional fp32 logits, NaN check, and the running argmax key of
// each token row. Thread = (token row, 32 vocabulary rows): the max over its 32
// keys, then over the four quarters, then one atomic per token row.
// one (token row m, 32 vocabulary rows) of the LM head: logits (optional), NaN check, key max
__device__ __forceinline__ unsigned long long argmax_item(const FwdArgs& a, const float* src, int m, int nt, int qq) {
  float y[32];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 f4 = *reinterpret_cast<const float4*>(src + 4 * c);
    y[4 * c] = f4.x, y[4 * c + 1] = f4.y, y[4 * c + 2] = f4.z, y[4 * c + 3] = f4.w;
  }
  const uint32_t col0 = nt * 128 + qq * 32;  // vocabulary index of y[0]
  unsigned long long best = 0ull;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool nan = isnan(y[i]);
    bad |= nan;
    best = ull_max(best, nan ? 0ull : argmax_key(y[i], col0 + i));
  }
  if (bad) set_status(a.status, ORTHRUS_ERR_NAN);
  if (a.logits) {
    float* lp = a.logits + (size_t)m * a.V + col0;
    if ((a.V & 3) == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        reinterpret_cast<float4*>(lp)[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) lp[i] = y[i];
    }
  }
  return best;
}

// Greedy head of the LM projection on token rows [m0, m0+32) (+ the second group v2) of one
// 128-row vocabulary tile: thread = (token row, 32 vocabulary rows), the max over its keys,
// then over the four quarters, then one atomic per token row. red: [128 + 16] keys.
__device__ __forceinline__ void fwd_argmax_epilogue(const FwdArgs& a, const float* v, const float* v2, int row, int m0,
                                                    int nt, int m_valid, float* epi, unsigned long long* red) {
  const int n2 = v2 ? epi_group2(m0, m_valid) : 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) epi[j * kEpiStride + row] = v[j];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < n2) epi[kEpi2 + k * kEpiStride + row] = v2[k];
  named_bar_sync(1, 128);
  const int t = threadIdx.x - 64, j = t & 31, qq = t >> 5;
  red[qq * 32 + j] = m0 + j < m_valid ? argmax_item(a, epi + j * kEpiStride + qq * 32, m0 + j, nt, qq) : 0ull;
  if (t < 4 * n2) {  // second group: thread = (row k, quarter q2)
    const int k = t >> 2, q2 = t & 3;
    red[128 + q2 * 4 + k] = argmax_item(a, epi + kEpi2 + k * kEpiStride + q2 * 32, m0 + 32 + k, nt, q2);
  }
  named_bar_sync(1, 128);
  if (t < 32 && m0 + t < m_valid) {
    const unsigned long long k = ull_max(ull_max(red[t], red[32 + t]), ull_max(red[64 + t], red[96 + t]));
    if (k != 0ull) atomicMax(a.amax + m0 + t, k);
  } else if (t >= 32 && t < 32 + n2) {
    const int k2 = t - 32;
    const unsigned long long k = ull_max(ull_max(red[128 + k2], red[132 + k2]), ull_max(red[136 + k2], red[140 + k2]));
    if (k != 0ull) atomicMax(a.amax + m0 + 32 + k2, k);
  }
}

// Epilogue of one 32-row group for the GEMM phase kinds. Consumers of a
// normalised input first scale by rstd of the token row.
template <int D_HEAD>
__device__ __forceinline__ void fwd_epilogue(const FwdArgs& a, const QkvCtx& qc, const int* lens_s,
                                             int epi_kind, float* v, float* v2, int row, int m0, int nt, int m_valid,
                                             float* epi, unsigned long long* red, const float* rstd_s,
                                             const float* gam_t, bool h_in_v = false) {
  if (epi_kind == EPI_RESID) {
    fwd_resid_epilogue(a, v, v2, row, m0, nt, m_valid, gam_t, epi, h_in_v);
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] *= rstd_s[m0 + j];
  if (v2) {
#pragma unroll
    for (int k = 0; k < 4; ++k) v2[k] *= rstd_s[m0 + 32 + k];
  }
  if (epi_kind == EPI_QKV) fwd_qkv_epilogue<D_HEAD>(a, qc, v, v2, row, m0, nt, m_valid, epi, lens_s);
  else if (epi_kind == EPI_SWIGLU) fwd_swiglu_epilogue(a, v, v2, row, m0, nt, m_valid, epi);
  else fwd_argmax_epilogue(a, v, v2, row, m0, nt, m_valid, epi, red);
}

}  // namespace orthrus

namespace orthrus {

// Accumulator columns [col, col + 32) (or + 4) of a projection. With two activation planes the
// MMA's N covers the Mt hi rows and then the Mt lo rows of the operand, so the lo products of
// token column j sit lo_off = Mt columns further on; they are added here (lo_off = 0: one plane).
__device__ __forceinline__ void acc_ld32(uint32_t taddr, int col, int lo_off, float* v) {
  tmem_ld32(taddr + col, v);
  if (lo_off) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float w[16];
      tmem_ld16(taddr + lo_off + col + 16 * h, w);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[16 * h + j] += w[j];
    }
  }
}

__device__ __forceinline__ void acc_ld4(uint32_t taddr, int col, int lo_off, float* v) {
  tmem_ld4(taddr + col, v);
  if (lo_off) {
    float w[4];
    tmem_ld4(taddr + lo_off + col, w);
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] += w[j];
  }
}

// Greedy consensus (verify launch) and counter reset; run by the last CTA to
// finish, when every other CTA has left the kernel.
__device__ inline void fwd_finalize(const FwdArgs& a, int n_ph) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  for (int m = t; m < a.M; m += blockDim.x) {
    const unsigned long long k = __ldcg(a.amax + m);
    int id = 0;
    if (k == 0ull) set_status(a.status, ORTHRUS_ERR_NAN);
    else id = (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    a.out_ids[m] = id;
  }
  __syncthreads();
  if (a.accept) {
    const bool err = *(volatile int*)a.status != 0;
    const int K = a.K;
    for (int b = warp; b < a.nb; b += blockDim.x >> 5) {
      // accept length = index of the first draft that differs from the AR argmax before it
      int acc = K;
      for (int i0 = 0; i0 < K; i0 += 32) {
        const int i = i0 + lane;
        const bool mism = i < K && a.draft_ids[b * K + i] != a.out_ids[b * (K + 1) + i];
        const unsigned bal = __ballot_sync(0xffffffffu, mism);
        if (bal) {
          acc = i0 + __ffs(bal) - 1;
          break;
        }
      }
      for (int i = lane; i <= K; i += 32) {
        int v = -1;
        if (!err && i < acc) v = a.draft_ids[b * K + i];
        else if (!err && i == acc) v = a.out_ids[b * (K + 1) + acc];
        a.committed[b * (K + 1) + i] = v;
      }
      if (lane == 0) {
        if (err) {
          a.accept_len[b] = -1;
        } else {
          a.accept_len[b] = acc;
          a.pending_out[b] = a.out_ids[b * (K + 1) + acc];
          a.len[b] += acc + 1;
        }
      }
    }
  }
  __syncthreads();
  for (int i = t; i < n_ph; i += blockDim.x) a.phase_cnt[i] = 0;
  if (t == 0) *a.exit_cnt = 0;
  __threadfence();
}

// Epilogue warps (2-5) of the persistent forward kernel. G2: the block has 33-36 token rows,
// whose rows past 32 ride with the first epilogue call (a separate instantiation, so blocks of
// at most 32 rows run without that code).
template <int D_HEAD, bool TL, bool G2>
__device__ __forceinline__ void fwd_epilogue_role(const FwdArgs& a, const FwdGeom& g, uint8_t* smem,
                                                  uint32_t stage_bytes, int S, uint8_t* scr,
                                                  unsigned long long* red, float* rstd_s, const int* lens_s,
                                                  const int* slot_pre, int* ust_s, uint64_t* accf, uint64_t* acce,
                                                  uint64_t* full, uint64_t* s_full, uint64_t* p_full,
                                                  uint64_t* o_full, int* flag,
                                                  uint32_t tmem_base, uint32_t tS, uint32_t tO) {
  constexpr int d = D_HEAD;
  constexpr int halves = d / 64;
  float* epi = (float*)scr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int et = threadIdx.x - 64;  // 0..127
  const int ew = warp - 2;          // 0..3
  const int quarter = warp & 3;     // TMEM lane quarter this warp may access
  const int row = quarter * 32 + lane;
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const int Gd = gridDim.x, c = blockIdx.x;
  const int n_ph = fwd_n_phases(a.L);
  const int D = a.D;
  int seg = 0, ta = 0, it = 0, acq = -1, bc = 0;
  bool ok = true;
  const uint64_t pol_keep = policy_evict_last();
  const uint64_t pol_drop = policy_evict_first();

  // one thread waits, the result is shared by the four warps (rotating flag slots
  // keep a slow reader from seeing the next call's value)
  auto bcast = [&](bool v_from_thread0) -> bool {
    const int slot = 1 + (bc++ & 3);
    if (et == 0) flag[slot] = v_from_thread0 ? 1 : 0;
    named_bar_sync(1, 128);
    return flag[slot] != 0;
  };
  int cur_p = 0;
  auto acquire_phase = [&](int dep) -> bool {
    if (dep <= acq) return true;
    bool r = false;
    if (et == 0) {
      const int tgt = phase_target(a, g, dep);
      const int code = wait_count_code(a.phase_cnt + dep, tgt, a.status, a.poll_ns);
      if (code == -1) fwd_diag(a, code, 12, cur_p, it, dep, tgt, *(volatile int*)(a.phase_cnt + dep));
      r = code == 1;
    }
    // thread 0's acquire, then the barrier in bcast: the other threads' later
    // reads are ordered after the released writes (happens-before is transitive)
    r = bcast(r);
    if (r) acq = dep;
    return r;
  };
  // outputs of a completion unit written -> count it (the barrier orders the other
  // threads' stores before thread 0's release, which is cumulative)
  auto signal = [&](int p, bool async_readers = true) {
    // the generic-proxy writes reach later TMA reads: proxy fence first (not needed when
    // every reader uses plain loads)
    if (async_readers) fence_proxy_async_global();
    named_bar_sync(1, 128);
    if (et == 0) red_release_gpu_add(a.phase_cnt + p, 1);
  };
  auto bar_wait_all = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
    bool r = false;
    if (et == 0) {
      const int code = mbar_wait_code(bar, parity, a.status);
      fwd_diag(a, code, site, cur_p, it, (int)parity, ta, seg);
      r = code == 1;
    }
    return bcast(r);
  };

  for (int p = 0; ok && p < n_ph; ++p) {
    const int kind = fwd_phase_kind(p, a.L);
    if (!phase_active(g, kind)) continue;
    const int l = fwd_phase_layer(p);
    const int dep = phase_dep(a, g, p);
    cur_p = p;

    if (kind == PH_EMBED) {
      // ---------------- embedding rows ----------------
      const float* g0 = a.norms[0].attn_norm;
      const int parts = D / 128;
      if (et == 0 && c < a.M) tl_mark<TL>(a, n_ph, p, TL_E0);
      for (int m = c; m < a.M; m += Gd) {
        const int bb = m / a.Q, i = m - bb * a.Q;
        int id;
        if (i == 0) id = a.pending[bb];
        else if (a.view == VIEW_VERIFY) id = a.draft_ids[bb * (a.Q - 1) + i - 1];
        else id = a.draft_ids ? a.draft_ids[bb * a.Q + i - 1] : a.mask_id;  // refinement: previous drafts
        if (id < 0 || id >= a.V) {
          if (et == 0) set_status(a.status, ORTHRUS_ERR_ARG);
          id = 0;
        }
        const int n = lens_s[bb];
        if (et == 0 && i == 0 && a.view == VIEW_VERIFY && n + a.Q > a.cap) set_status(a.status, ORTHRUS_ERR_CAPACITY);
        const __nv_bfloat16* src = a.embed + (size_t)id * D;
        for (int pp = 0; pp < parts; ++pp) {
          const int col = pp * 128 + et;
          const float x = __bfloat162float(src[col]);
          a.h[(size_t)m * D + col] = x;
          const float xv = x * g0[col];
          const __nv_bfloat16 xh = __float2bfloat16(xv);
          a.xg[(size_t)m * D + col] = xh;
          a.xg[a.xg_lo + (size_t)m * D + col] = __float2bfloat16(xv - __bfloat162float(xh));
          const float s = warp_sum(x * x);
          if (lane == 0) epi[ew * 64 + pp] = s;
        }
        named_bar_sync(1, 128);
        if (et < parts) a.ss[(size_t)et * a.ss_ld + m] = ((epi[et] + epi[64 + et]) + epi[128 + et]) + epi[192 + et];
        if (et < d / 2) {
          const double ang = (double)(n + i) * pow(a.theta, -2.0 * (double)et / (double)d);
          a.rope[(size_t)m * (d / 2) + et] = make_float2((float)cos(ang), (float)sin(ang));
        }
        if (et == 0) a.amax[m] = 0ull;
        named_bar_sync(1, 128);
        signal(p);
      }
    } else if (is_gemm_kind(kind)) {
      // ---------------- projection epilogues ----------------
      const GemmPhase gp = gemm_phase(a, kind, l);
      const long long W = gp.units;
      const long long u0 = unit_start(W, Gd, c), u1 = unit_start(W, Gd, c + 1);
      const int kc = gp.k_chunks;
      if (u0 == u1) continue;
      // unit-range start of every CTA (W * Gd < 2^31 for every phase shape accepted)
      for (int i = et; i <= Gd; i += 128) ust_s[i] = (int)(((long long)W * i) / Gd);
      const int first_tile = (int)(u0 / kc), last_tile = (int)((u1 - 1) / kc);
      // Per-phase epilogue inputs are copied to the attention Q region (unused by
      // projection phases): QKV: q/k norm gains and RoPE rows; O / DOWN: the next norm's
      // gains of the CTA's tiles. Weights are copied before the previous phase is
      // awaited (RoPE rows too, once EMBED is long done), each thread's loads all in
      // flight before its shared-memory stores.
      float* stg = reinterpret_cast<float*>(scr - (size_t)128 * d * 2);
      const int stg_floats = 64 * d;
      const float* gam = nullptr;
      bool gam_staged = false;
      QkvCtx qc;
      qc.kdst = qc.vdst = nullptr;
      qc.kv_stride = 0;
      qc.gains = stg;
      qc.rope = reinterpret_cast<const float2*>(stg + 2 * d);
      qc.rope_rows = 0;
      // RoPE rows [0, rope_rows) -> shared memory, 16-byte chunk c of segment s at chunk
      // s*8 + ((c + 2s + (m & 1)) & 7) of the row (conflict-free reads in the epilogue)
      auto stage_rope = [&]() {
        const float4* rs = reinterpret_cast<const float4*>(a.rope);
        float4* rd = reinterpret_cast<float4*>(stg + 2 * d);
        const int n = qc.rope_rows * (d / 4);  // a row is d/2 float2 = d/4 16-byte chunks
        for (int b0 = 0; b0 < n; b0 += 128 * 8) {
          float4 buf[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int i = b0 + et + 128 * k;
            buf[k] = i < n ? __ldcg(rs + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int i = b0 + et + 128 * k;
            if (i < n) {
              const int m = i / (d / 4), kk = i - m * (d / 4), sg = kk >> 3, cc = kk & 7;
              rd[m * (d / 4) + sg * 8 + ((cc + 2 * sg + (m & 1)) & 7)] = buf[k];
            }
          }
        }
      };
      if (kind == PH_QKV) {
        const bool dv = a.view == VIEW_DRAFT;
        const float4* gq = reinterpret_cast<const float4*>(dv ? a.norms[l].wd_q_norm : a.norms[l].q_norm);
        const float4* gk = reinterpret_cast<const float4*>(dv ? a.norms[l].wd_k_norm : a.norms[l].k_norm);
        if (et < d / 2) {  // d/4 float4 of q gains, then d/4 of k gains
          const float4* src = et < d / 4 ? gq + et : gk + (et - d / 4);
          const float4 g4 = a.qk_norm ? *src : make_float4(1.f, 1.f, 1.f, 1.f);
          reinterpret_cast<float4*>(stg)[et] = g4;
        }
        qc.rope_rows = min(a.M, (stg_floats - 2 * d) / d);
        if (l > 0) stage_rope();
        if (dv) {
          const size_t lo = (size_t)l * a.batch * a.Hkv * a.max_block * d;
          qc.kdst = a.blk_k + lo;
          qc.vdst = a.blk_v + lo;
          qc.kv_stride = a.max_block;
        } else {
          const size_t lo = (size_t)l * a.batch * a.Hkv * a.cap * d;
          qc.kdst = a.kc + lo;
          qc.vdst = a.vc + lo;
          qc.kv_stride = a.cap;
        }
      } else if (kind == PH_O || kind == PH_DOWN) {
        gam = kind == PH_O ? a.norms[l].mlp_norm : (l + 1 < a.L ? a.norms[l + 1].attn_norm : a.final_norm);
        const int n4 = (last_tile - first_tile + 1) * 32;  // float4 of gains
        if (n4 * 4 <= stg_floats) {
          const float4* src = reinterpret_cast<const float4*>(gam + (size_t)first_tile * 128);
          for (int b0 = 0; b0 < n4; b0 += 128 * 4) {
            float4 buf[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = b0 + et + 128 * k;
              buf[k] = i < n4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = b0 + et + 128 * k;
              if (i < n4) reinterpret_cast<float4*>(stg)[i] = buf[k];
            }
          }
          gam_staged = true;
        }
      }
      if (!acquire_phase(dep)) {
        ok = false;
        break;
      }
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E0);
      if (kind == PH_QKV && l == 0) stage_rope();  // written by EMBED in this launch
      if (kind == PH_QKV || kind == PH_GU || kind == PH_LM) {
        // rstd of every token row from the D/128 per-tile sums of squares: thread (row m,
        // quarter q) adds every fourth partial (its loads all in flight at once), then the
        // four quarters are added in a fixed order
        const int np = D / 128;
        for (int m0 = 0; m0 < a.Mt; m0 += 32) {
          const int m = m0 + (et & 31), q = et >> 5;
          float s = 0.f;
          if (m < a.M) {
#pragma unroll 8
            for (int pp = q; pp < np; pp += 4) s += __ldcg(a.ss + (size_t)pp * a.ss_ld + m);
          }
          epi[et] = s;
          named_bar_sync(1, 128);
          if (q == 0 && m < a.Mt)
            rstd_s[m] = m < a.M ? rsqrtf((((epi[et] + epi[32 + et]) + epi[64 + et]) + epi[96 + et]) / (float)D + a.eps)
                                : 0.f;
          named_bar_sync(1, 128);
        }
      }
      named_bar_sync(1, 128);
      auto gam_tile = [&](int t) -> const float* {
        if (!gam) return nullptr;
        return gam_staged ? stg + (t - first_tile) * 128 : gam + (size_t)t * 128;
      };
      const int m_valid = min(a.Mt, a.M);
      const int n2 = G2 ? epi_group2(0, m_valid) : 0;  // rows past 32 that ride with the first call
      // owner of unit uu = the CTA whose non-empty range holds it (largest c with start <= uu)
      auto owner = [&](int uu) {
        int lo = 0, hi = Gd - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (ust_s[mid] <= uu) lo = mid;
          else hi = mid - 1;
        }
        return lo;
      };
      // partial slot of contributor cc to tile t: its first or its last segment
      auto part_slot = [&](int cc, int t) { return 2 * cc + (ust_s[cc] / kc == t ? 0 : 1); };
      // next (up to) two non-empty contributors from cc on, in k order (two per round: four
      // rounds' worth of prefetched partials cost registers the rest of the kernel needs)
      auto gather2 = [&](int& cc, int c_hi, int& s0, int& s1, int t) {
        s0 = s1 = -1;
        for (int q = 0; q < 2 && cc <= c_hi; ++cc) {
          if (ust_s[cc + 1] > ust_s[cc]) {
            const int sl = part_slot(cc, t);
            if (q == 0) s0 = sl;
            else s1 = sl;
            ++q;
          }
        }
      };
      auto load2 = [&](float4 (&x)[2][8], int s0, int s1, int m0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int sl = q == 0 ? s0 : s1;
          const float4* pp = reinterpret_cast<const float4*>(a.partial + (size_t)(sl < 0 ? 0 : sl) * (128 * 128)) +
                             (size_t)(m0 >> 2) * 128 + row;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            x[q][q4] = (sl >= 0 && m0 + 4 * q4 < m_valid) ? ld_f4_hint(pp + (size_t)q4 * 128, pol_drop)
                                                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      };
      auto add2 = [&](float* v, const float4 (&x)[2][8]) {
#pragma unroll
        for (int q = 0; q < 2; ++q)  // fixed k order within and across rounds
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            v[4 * q4] += x[q][q4].x;
            v[4 * q4 + 1] += x[q][q4].y;
            v[4 * q4 + 2] += x[q][q4].z;
            v[4 * q4 + 3] += x[q][q4].w;
          }
      };
      long long u = u0;
      while (ok && u < u1) {
        const int t = (int)(u / kc);
        const long long seg_start = u, seg_end = min(u1, (long long)(t + 1) * kc);
        u = seg_end;
        const int buf = seg & 1, use = seg >> 1;
        ++seg;
        const int nt = t;
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * 256;
        const int lo_off = gp.planes == 2 ? a.Mt : 0;
        const bool whole = seg_start == (long long)t * kc && seg_end == (long long)(t + 1) * kc;
        float v[32];
        if (whole) {
          if (!bar_wait_all(&accf[buf], (uint32_t)use & 1u, 13)) {
            ok = false;
            break;
          }
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_ACC);
          tc_fence_after();
          for (int m0 = 0; m0 < a.Mt; m0 += 32) {
            if (m0 == 32 && n2 > 0) break;  // rows 32.. went with the first call
            acc_ld32(taddr, m0, lo_off, v);
            float v2[4];
            if (m0 == 0 && n2 > 0) acc_ld4(taddr, 32, lo_off, v2);
            fwd_epilogue<D_HEAD>(a, qc, lens_s, gp.epi, v, m0 == 0 && n2 > 0 ? v2 : nullptr, row, m0, nt, m_valid,
                                 epi, red, rstd_s, gam_tile(nt));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[buf]);
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_EPI);
          signal(p);
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_SIG);
          continue;
        }
        const int c_lo = owner(t * kc), c_hi = owner((t + 1) * kc - 1);
        // The tile's head owner c_lo (it holds the first k unit) finishes the tile: the
        // other contributors release a count after storing their partial, c_lo waits
        // for all of them. A CTA is head owner of at most one split tile (its last
        // segment), so no CTA runs two fixups in a row. Waits point only to higher-indexed
        // CTAs, whose parts are stored (their first segment) before they wait on anything.
        const bool head = c == c_lo;
        if (!head) {
          if (!bar_wait_all(&accf[buf], (uint32_t)use & 1u, 13)) {
            ok = false;
            break;
          }
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_ACC);
          tc_fence_after();
          const bool add_h = gp.epi == EPI_RESID && c == c_hi;
          // partial slot layout [token m / 4][weight row][m % 4]: a thread moves float4s and a
          // warp's access is 512 contiguous bytes
          const int slot = 2 * c + (t == first_tile ? 0 : 1);
          float4* part = reinterpret_cast<float4*>(a.partial + (size_t)slot * (128 * 128)) + row;
          for (int m0 = 0; m0 < a.Mt; m0 += 32) {
            acc_ld32(taddr, m0, lo_off, v);
            if (add_h) {
              float hv[32];
#pragma unroll
              for (int j = 0; j < 32; ++j)
                hv[j] = (m0 + j < m_valid) ? __ldcg(a.h + (size_t)(m0 + j) * D + nt * 128 + row) : 0.f;
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += hv[j];
            }
            // partials stay in L2 (evict_last) while the weight stream passes through it
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              if (m0 + 4 * q4 < m_valid)  // only token columns that exist
                st_f4_hint(part + (size_t)((m0 >> 2) + q4) * 128,
                           make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]), pol_keep);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[buf]);
          named_bar_sync(1, 128);
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_PART);
          if (et == 0) red_release_gpu_add(a.tile_cnt + t, 1);
          continue;
        }
        // Head owner. The other contributors stored their parts at the start of their
        // ranges, long before this CTA's own part (the end of its range) is accumulated:
        // their count is awaited and the first token group of all of them summed, in k
        // order, while the MMAs of the last k units still run; only the add of that sum
        // to the own part is left for when the accumulator is ready.
        int n_contrib = 0;
        for (int cc = c_lo; cc <= c_hi; ++cc) n_contrib += ust_s[cc + 1] > ust_s[cc];
        bool ready = false;
        if (et == 0) {
          const int code = wait_count_code(a.tile_cnt + t, n_contrib - 1, a.status);
          if (code == -1) fwd_diag(a, code, 17, p, it, t, n_contrib, *(volatile int*)(a.tile_cnt + t));
          ready = code == 1;
          if (ready) a.tile_cnt[t] = 0;
        }
        if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_CNT);
        if (!bcast(ready)) {
          ok = false;
          break;
        }
        // pre = c_lo+1 + c_lo+2 + ... + c_hi (token rows 0..31, and the second group's rows
        // 32..35 when they ride with the first call); the own part is added to it last
        float pre[32], pre2[4];
#pragma unroll
        for (int j = 0; j < 32; ++j) pre[j] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) pre2[k] = 0.f;
        for (int cc = c_lo + 1; cc <= c_hi;) {
          int s0, s1;
          gather2(cc, c_hi, s0, s1, t);
          float4 x[2][8];
          load2(x, s0, s1, 0);
          float4 x2[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int sl = q == 0 ? s0 : s1;
            x2[q] = (sl >= 0 && n2 > 0)
                        ? ld_f4_hint(reinterpret_cast<const float4*>(a.partial + (size_t)sl * (128 * 128)) + 8 * 128 +
                                         row,
                                     pol_drop)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          add2(pre, x);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            pre2[0] += x2[q].x;
            pre2[1] += x2[q].y;
            pre2[2] += x2[q].z;
            pre2[3] += x2[q].w;
          }
        }
        if (!bar_wait_all(&accf[buf], (uint32_t)use & 1u, 13)) {
          ok = false;
          break;
        }
        if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_ACC);
        tc_fence_after();
        for (int m0 = 0; m0 < a.Mt; m0 += 32) {
          if (m0 == 32 && n2 > 0) break;  // rows 32.. went with the first call
          const bool fuse = m0 == 0 && n2 > 0;
          acc_ld32(taddr, m0, lo_off, v);  // own part: the first k units of the tile
          float v2[4];
          if (fuse) acc_ld4(taddr, 32, lo_off, v2);
          if (m0 == 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += pre[j];
            if (fuse) {
#pragma unroll
              for (int k = 0; k < 4; ++k) v2[k] += pre2[k];
            }
          } else {
            // further token groups (blocks of more than 36 rows): the contributors in the same
            // k order, summed first as for the first group, then added to the own part
            float sum[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[j] = 0.f;
            for (int cc = c_lo + 1; cc <= c_hi;) {
              int s0, s1;
              gather2(cc, c_hi, s0, s1, t);
              float4 x[2][8];
              load2(x, s0, s1, m0);
              add2(sum, x);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += sum[j];
          }
          if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_LOAD);
          fwd_epilogue<D_HEAD>(a, qc, lens_s, gp.epi, v, fuse ? v2 : nullptr, row, m0, nt, m_valid, epi, red, rstd_s,
                               gam_tile(nt), true);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[buf]);
        if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_EPI);
        signal(p);
        if (et == 0) tl_mark<TL>(a, n_ph, p, TL_S_SIG);
      }
      it += (int)(u1 - u0);
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E1);
    } else if (kind == PH_ATTN) {
      // ---------------- block attention (thread = query row of the tile) ----------------
      if (c >= g.att_units) continue;
      if (!acquire_phase(dep)) {
        ok = false;
        break;
      }
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E0);
      for (int u = c; ok && u < g.att_units; u += Gd) {
        const AttUnit t = att_unit(a, g, lens_s, slot_pre, u);
        const int grow = t.r * 128 + row;
        const bool row_ok = grow < g.rows_per_slot;
        const int i = row_ok ? grow / a.G : 0;
        const int row_hi = min(g.rows_per_slot, (t.r + 1) * 128);
        const int i_max = (row_hi - 1) / a.G;
        int lim = t.key_hi, kv_end = t.key_hi;
        if (a.view == VIEW_VERIFY) {
          lim = min(t.n + i + 1, t.key_hi);
          kv_end = min(t.n + i_max + 1, t.key_hi);
        }
        if (!row_ok) lim = t.key_lo;
        // O accumulates in TMEM across the unit's key tiles (P V MMAs with accumulate);
        // when a row's exponent offset moves (below), the row of O is rescaled in TMEM
        // before the next P V. O is read into registers once, after the last tile. P of a
        // tile sits beside its V in the ring stage, so P of the next tile can be written
        // while this tile's P V still reads.
        float m_run = -INFINITY, l_run = 0.f;
        for (int j = 0; j < t.tiles; ++j, ++it, ++ta) {
          // score buffer ta & 1; its barrier completes once per use, every second tile
          if (!bar_wait_all(&s_full[(ta & 1) * 3], (uint32_t)(ta >> 1) & 1u, 14)) {
            ok = false;
            break;
          }
          const uint32_t tSb = (ta & 1) ? tS + 192 : tS;  // the second buffer sits at column 448
          if (et == 0) tl_mark<TL>(a, n_ph, p, j == 0 ? TL_R0 : TL_S_ACC);  // score tile ready
          tc_fence_after();
          const int key0 = t.key_lo + j * 64;
          const int nv = min(max(lim - key0, 0), 64);  // keys of this tile the row sees
          // Row maximum over the visible scores: two 32-column loads, four independent
          // chains (the scale is positive, so max(s) * scale = max(s * scale) exactly).
          // The scores are loaded again for the exponentials below rather than held:
          // fewer live registers leave room for independent work in both passes.
          float sv[32];
          float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            tmem_ld32(tSb + lane_base + c0, sv);
#pragma unroll
            for (int tt = 0; tt < 32; tt += 4) {
              mx0 = fmaxf(mx0, c0 + tt < nv ? sv[tt] : -INFINITY);
              mx1 = fmaxf(mx1, c0 + tt + 1 < nv ? sv[tt + 1] : -INFINITY);
              mx2 = fmaxf(mx2, c0 + tt + 2 < nv ? sv[tt + 2] : -INFINITY);
              mx3 = fmaxf(mx3, c0 + tt + 3 < nv ? sv[tt + 3] : -INFINITY);
            }
          }
          const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * a.scale_log2;
          // The exponent offset m_run moves only when a score passes it by more than
          // kRescaleLog2 (then the weights below stay under 2^kRescaleLog2, well inside fp16),
          // so O is rarely rescaled and this tile's softmax need not wait for the previous P V.
          const bool grow = mx > m_run + kRescaleLog2;
          const float m_new = grow ? mx : m_run;
          const float alpha = (grow && m_run != -INFINITY) ? fast_exp2(m_run - m_new) : 1.f;
          if (j == 0 && et == 0) tl_mark<TL>(a, n_ph, p, TL_S_PART);  // row maxima done
          // this tile's stage: K, V, then P. Its K and V landed before S was issued, and the
          // P region's previous reader released the stage before they were loaded.
          const int vs = it % S;
          if (j > 0 && named_bar_or(1, 128, alpha != 1.f)) {
            // the previous tile's P V must be complete before O is rescaled
            if (!bar_wait_all(&o_full[(ta - 1) & 1], (uint32_t)((ta - 1) >> 1) & 1u, 15)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {  // warp-uniform: tcgen05.ld/st are per warp
#pragma unroll
              for (int c0 = 0; c0 < d; c0 += 32) {
                float v[32];
                tmem_ld32(tO + lane_base + c0, v);
#pragma unroll
                for (int tt = 0; tt < 32; ++tt) v[tt] *= alpha;
                tmem_st32(tO + lane_base + c0, v);
              }
            }
          }
          uint8_t* vb = smem + (size_t)vs * stage_bytes + halves * 8192;  // V, then P
          float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            tmem_ld32(tSb + lane_base + c0, sv);
            uint32_t pk[16];
#pragma unroll
            for (int tt = 0; tt < 32; tt += 2) {
              // masked keys get exp2(-inf) = 0: the select is on the argument, so no branch
              // surrounds the (asm) exponential and the 32 of them can overlap
              const float p0 = fast_exp2(c0 + tt < nv ? sv[tt] * a.scale_log2 - m_new : -INFINITY);
              const float p1 = fast_exp2(c0 + tt + 1 < nv ? sv[tt + 1] * a.scale_log2 - m_new : -INFINITY);
              sum0 += p0;
              sum1 += p1;
              __half2 h2 = __floats2half2_rn(p0, p1);
              pk[tt / 2] = *reinterpret_cast<uint32_t*>(&h2);
            }
            uint8_t* rowp = vb + halves * 8192 + row * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int ch = (c0 >> 3) + q4;
              *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) =
                  make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            }
          }
          l_run = l_run * alpha + (sum0 + sum1);
          m_run = m_new;
          // V rows of keys no row may see are zeroed (stale or poisoned cache rows); the wait
          // orders these writes after the TMA's
          if (key0 + 64 > kv_end && row < 64 && key0 + row >= kv_end &&
              mbar_wait_abortable(&full[vs], (uint32_t)(it / S) & 1u, a.status)) {
#pragma unroll
            for (int hh = 0; hh < halves; ++hh) {
              uint4* vr = reinterpret_cast<uint4*>(vb + hh * 8192 + row * 128);
#pragma unroll
              for (int q8 = 0; q8 < 8; ++q8) vr[q8] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[ta & 1]);
          if (j == 0 && et == 0) tl_mark<TL>(a, n_ph, p, TL_S_CNT);  // P written
        }
        if (!ok) break;
        // the unit's last P V, then O into registers
        if (!bar_wait_all(&o_full[(ta - 1) & 1], (uint32_t)((ta - 1) >> 1) & 1u, 15)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float o[d];
#pragma unroll
        for (int c0 = 0; c0 < d; c0 += 32) tmem_ld32(tO + lane_base + c0, o + c0);
        tc_fence_before();
        if (et == 0) tl_mark<TL>(a, n_ph, p, TL_R1);
        const int H = a.H;
        if (t.n_chunks == 1) {
          if (row_ok) {
            const int gg = grow - i * a.G;
            __nv_bfloat16* dst = a.attn + ((size_t)(t.bb * a.Q + i) * H + t.kvh * a.G + gg) * d;
            const float inv = l_run > 0.f ? __fdividef(1.f, l_run) : 0.f;
#pragma unroll
            for (int e = 0; e < d; e += 8) {
              float y8[8];
#pragma unroll
              for (int tt = 0; tt < 8; ++tt) y8[tt] = o[e + tt] * inv;
              st_split_x8(dst + e, dst + a.attn_lo + e, y8);
            }
          }
        } else {
          // partial O in a [chunk][d/4][row][4] layout: a warp's float4 stores are 512 contiguous bytes
          const size_t pidx = ((size_t)t.slot * kMaxChunks + t.chunk) * 128 + row;
          float4* po = reinterpret_cast<float4*>(a.att_o) + ((size_t)t.slot * kMaxChunks + t.chunk) * (d / 4) * 128 + row;
#pragma unroll
          for (int e = 0; e < d; e += 4) __stcg(po + (size_t)(e / 4) * 128, make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]));
          __stcg(a.att_ml + pidx, make_float2(m_run, l_run));
        }
        signal(p, t.n_chunks == 1);  // partials are read by the merge with plain loads
      }
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E1);
    } else if (kind == PH_COMBINE) {
      // ---------------- merge of key-chunk partials ----------------
      if (c >= g.comb_units) continue;
      if (!acquire_phase(dep)) {
        ok = false;
        break;
      }
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E0);
      constexpr int per = d / 8;  // columns per thread: thread et takes row et % 16 and column block et / 16
      for (int u = c; u < g.comb_units; u += Gd) {
        const int slot = u / (128 / kCombineRows), grp = u % (128 / kCombineRows);
        const int nch = slot_pre[slot + 1] - slot_pre[slot];
        const int r_t = slot % g.rt, kvh = (slot / g.rt) % a.Hkv, bb = slot / (g.rt * a.Hkv);
        const int r = grp * kCombineRows + (et & 15), sub = et >> 4;
        const int grow = r_t * 128 + r;
        if (nch > 1 && grow < g.rows_per_slot) {
          const int i = grow / a.G, gg = grow - i * a.G;
          const float2* ml = a.att_ml + (size_t)slot * kMaxChunks * 128 + r;
          // online merge over batches of up to 8 chunks: a batch's (m, l) and O loads are all
          // in flight together; the running maximum rescales the sums between batches
          float mrun = -INFINITY, L = 0.f;
          float acc[per];
#pragma unroll
          for (int e = 0; e < per; ++e) acc[e] = 0.f;
          for (int c0 = 0; c0 < nch; c0 += 8) {
            float2 mlb[8];
            float4 ob[8][per / 4];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const bool in = c0 + k < nch;
              mlb[k] = in ? __ldcg(ml + (c0 + k) * 128) : make_float2(-INFINITY, 0.f);
              const float4* po = reinterpret_cast<const float4*>(a.att_o) +
                                 (((size_t)slot * kMaxChunks + (in ? c0 + k : 0)) * (d / 4) + sub * (per / 4)) * 128 + r;
#pragma unroll
              for (int e = 0; e < per / 4; ++e) ob[k][e] = in ? __ldcg(po + (size_t)e * 128) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float mb = mrun;
#pragma unroll
            for (int k = 0; k < 8; ++k) mb = fmaxf(mb, mlb[k].x);
            if (mb != -INFINITY) {
              const float sc = mrun == -INFINITY ? 0.f : fast_exp2(mrun - mb);
              L *= sc;
#pragma unroll
              for (int e = 0; e < per; ++e) acc[e] *= sc;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float w = mlb[k].x == -INFINITY ? 0.f : fast_exp2(mlb[k].x - mb);
                L += w * mlb[k].y;
#pragma unroll
                for (int e = 0; e < per / 4; ++e) {
                  acc[4 * e] += w * ob[k][e].x;
                  acc[4 * e + 1] += w * ob[k][e].y;
                  acc[4 * e + 2] += w * ob[k][e].z;
                  acc[4 * e + 3] += w * ob[k][e].w;
                }
              }
              mrun = mb;
            }
          }
          const float inv = L > 0.f ? __fdividef(1.f, L) : 0.f;
          __nv_bfloat16* dst = a.attn + ((size_t)(bb * a.Q + i) * a.H + kvh * a.G + gg) * d + sub * per;
#pragma unroll
          for (int e = 0; e < per; e += 8) {
            float y8[8];
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) y8[tt] = acc[e + tt] * inv;
            st_split_x8(dst + e, dst + a.attn_lo + e, y8);
          }
        }
        signal(p);
      }
      if (et == 0) tl_mark<TL>(a, n_ph, p, TL_E1);
    }
  }
}

}  // namespace orthrus

namespace orthrus {

template <int D_HEAD, bool TL, bool G2>
__global__ void __launch_bounds__(kFwdThreads, 1) forward_kernel(const __grid_constant__ FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int d = D_HEAD;
  constexpr int halves = d / 64;
  const int S = a.stages;
  const uint32_t stage_bytes = fwd_stage_bytes(a.Mt, d);
  uint8_t* sQ = smem + (size_t)S * stage_bytes;   // attention Q tile, d/64 blocks of 128 rows x 64
  uint8_t* scr = sQ + (size_t)128 * d * 2;         // epilogue staging
  unsigned long long* red = (unsigned long long*)(scr + kScratchBytes);
  float* rstd_s = (float*)(red + 144);
  int* lens_s = (int*)(rstd_s + 128);
  int* slot_pre = lens_s + 128;
  int* ust_s = slot_pre + kMaxSlots + 1;  // [grid + 1] unit-range starts of the current phase
  uint64_t* bars = (uint64_t*)(((uintptr_t)(ust_s + kMaxGrid) + 7) & ~(uintptr_t)7);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxStages;
  uint64_t* accf = bars + 2 * kMaxStages;  // [2]
  uint64_t* acce = accf + 2;               // [2]
  uint64_t* s_full = acce + 2;  // [0] and [3]: scores of even / odd key tiles ready
  uint64_t* done = s_full + 4;
  uint64_t* q_full = s_full + 5;
  uint64_t* q_empty = s_full + 6;
  uint64_t* p_full = s_full + 7;  // [2]: P of even / odd key tiles written
  uint64_t* o_full = s_full + 9;  // [2]: P V of even / odd key tiles done
  uint32_t* tmem_slot = (uint32_t*)(s_full + 11);
  int* flag = (int*)(tmem_slot + 1);  // [8]
  FwdGeom* geom_s = (FwdGeom*)(flag + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Gd = gridDim.x, c = blockIdx.x;
  const int n_ph = fwd_n_phases(a.L);
  auto stage_ptr = [&](int s) { return smem + (size_t)s * stage_bytes; };

  // ---------------- set-up ----------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 2);  // one arrival from each producer
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(s_full, 1);
    mbar_init(s_full + 3, 1);  // second score buffer
    for (int b = 0; b < 2; ++b) {
      mbar_init(&p_full[b], 4);
      mbar_init(&o_full[b], 1);
    }
    mbar_init(done, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < a.nb) lens_s[threadIdx.x] = a.len[threadIdx.x];
  __syncthreads();
  if (warp == 0) {
    FwdGeom g;
    g.rows_per_slot = a.Q * a.G;
    g.rt = (g.rows_per_slot + 127) / 128;
    g.slots = a.nb * a.Hkv * g.rt;
    g.CK = a.ck;
    if (a.view == VIEW_DRAFT) {
      // The verify view keeps the plan's chunk length, so that its rows and plain decoding
      // see the same chunk boundaries. The draft view's rows are matched with no other
      // launch, so its chunks are the shortest whose units (one per chunk, plus the block)
      // fit one wave of CTAs for the current cache lengths: lane j tries ck0 + 64 j.
      int n_max = 0;
      for (int bb = lane; bb < a.nb; bb += 32) n_max = max(n_max, min(lens_s[bb], a.cap));
      for (int o = 16; o > 0; o >>= 1) n_max = max(n_max, __shfl_xor_sync(0xffffffffu, n_max, o));
      const int ck0 = max(64, ((n_max + 31) / 32 + 63) / 64 * 64);  // at most 32 cache chunks
      const int ck = ck0 + 64 * lane;
      long long units = 0;
      for (int bb = 0; bb < a.nb; ++bb)
        units += (long long)a.Hkv * g.rt * ((min(lens_s[bb], a.cap) + ck - 1) / ck + 1);
      const unsigned fit = __ballot_sync(0xffffffffu, ck < a.ck && units <= Gd);
      if (fit) g.CK = ck0 + 64 * (__ffs((int)fit) - 1);
    }
    if (lane == 0) {
      slot_pre[0] = 0;
      bool multi = false;
      for (int s = 0; s < g.slots; ++s) {
        const int ch = slot_chunks(a, g, lens_s, s);
        multi = multi || ch > 1;
        slot_pre[s + 1] = slot_pre[s] + ch;
      }
      g.att_units = slot_pre[g.slots];
      g.comb_units = multi ? g.slots * (128 / kCombineRows) : 0;
      *geom_s = g;
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const FwdGeom g = *geom_s;
  const uint32_t tmem_base = *tmem_slot;
  // TMEM: two projection accumulators of up to 256 columns (2 Mt: hi and lo products) at 0 and 256.
  // The attention tiles alias the second one: a projection accumulator is read by its epilogue
  // before the phase completes, and attention MMAs wait for the q/k/v phase's completion (the Q
  // tile); the next projection's MMAs wait for the attention phase's output (their activations).
  const uint32_t tS = tmem_base + 256;   // attention scores: 64 columns (even key tiles)
  const uint32_t tO = tmem_base + 320;   // attention P V tile: d columns
  const uint32_t tS2 = tmem_base + 448;  // scores of odd key tiles

  if (warp == 0 || warp == 6) {
    // ============ TMA producers: warp 0 streams weight tiles, warp 6 activations ============
    // Both walk the same ring; a stage's full barrier expects one arrival from each.
    // The weight producer never waits for a dependency, so it runs up to a ring ahead
    // into the next phase while the activation producer waits for the phase before.
    if (lane == 0) {
      const bool wprod = warp == 0;
      const CUtensorMap* gm = a.maps + (size_t)a.L * M_PER_LAYER;
      const uint64_t pol_w = policy_evict_first();
      int last_ph[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last_ph[s] = -1;
      int known_done = -1;
      bool ok = true;
      int it = 0, qu = 0;
      int cur_p = 0;
      auto dep_ready = [&](int dep) -> bool {
        if (dep <= known_done) return true;
        const int tgt = phase_target(a, g, dep);
        const int r = wait_count_code(a.phase_cnt + dep, tgt, a.status, a.poll_ns);
        if (r != 1) {
          fwd_diag(a, r, 3, cur_p, it, dep, tgt, *(volatile int*)(a.phase_cnt + dep));
          return false;
        }
        known_done = dep;
        fence_proxy_async_global();
        return true;
      };
      for (int p = 0; ok && p < n_ph; ++p) {
        const int kind = fwd_phase_kind(p, a.L);
        if (!phase_active(g, kind)) continue;
        const int l = fwd_phase_layer(p);
        const int dep = phase_dep(a, g, p);
        cur_p = p;
        if (is_gemm_kind(kind)) {
          const GemmPhase gp = gemm_phase(a, kind, l);
          const long long W = gp.units;
          const long long u0 = unit_start(W, Gd, c), u1 = unit_start(W, Gd, c + 1);
          const int kc = gp.k_chunks;
          if (u0 < u1 && wprod) tl_mark<TL>(a, n_ph, p, TL_W0);
          for (long long u = u0; u < u1; ++u, ++it) {
            const int s = it % S;
            const uint32_t ph = (uint32_t)(it / S) & 1u;
            const int r = mbar_wait_code(&empty[s], ph ^ 1u, a.status);
            if (r != 1) {
              fwd_diag(a, r, wprod ? 1 : 2, p, it, s);
              ok = false;
              break;
            }
            const int t = (int)(u / kc), k = (int)(u - (long long)t * kc);
            uint8_t* st = stage_ptr(s);
            if (wprod) {
              // run ahead into a phase whose input is not ready by at most `lookahead` tiles
              if (u - u0 >= a.lookahead && !dep_ready(dep)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&full[s], 32768u);
              if (gp.gu) tma_load_4d_hint(st, gp.mw, &full[s], 0, t * 64, 0, 2 * k, pol_w);  // gate + up rows
              else tma_load_3d_hint(st, gp.mw, &full[s], 0, t * 128, 2 * k, pol_w);
            } else {
              if (!dep_ready(dep)) {
                ok = false;
                break;
              }
              if (u == u0) tl_mark<TL>(a, n_ph, p, TL_X0);
              // box [k chunk][plane][Mt rows][64] (one plane for the LM head)
              mbar_arrive_expect_tx(&full[s], (uint32_t)a.Mt * 256u * (uint32_t)gp.planes);
              if (gp.planes == 2) tma_load_4d(st + 32768, gp.mx, &full[s], 0, 0, 0, 2 * k);
              else tma_load_3d(st + 32768, gp.mx, &full[s], 0, 0, 2 * k);
            }
            last_ph[s] = (int)ph;
          }
          if (u0 < u1) tl_mark<TL>(a, n_ph, p, wprod ? TL_W1 : TL_X1);
        } else if (kind == PH_ATTN) {
          for (int u = c; ok && u < g.att_units; u += Gd, ++qu) {
            const AttUnit t = att_unit(a, g, lens_s, slot_pre, u);
            const int zc = (l * a.batch + t.bb) * a.Hkv + t.kvh;
            const int qrow = (t.bb * a.Hkv + t.kvh) * g.rows_per_slot + t.r * 128;
            // Cache keys below len were written by earlier launches: their K/V tiles are
            // loaded without waiting for this layer's q/k/v phase. The Q tile and block
            // keys wait for it; Q goes out before the first such load, or after the first
            // K/V tile when that tile is independent.
            bool q_issued = false;
            auto issue_q = [&]() -> bool {
              if (!dep_ready(dep)) return false;
              mbar_arrive_expect_tx(q_full, 16384u * halves);
              for (int hh = 0; hh < halves; ++hh) tma_load_2d(sQ + hh * 16384, gm + G_Q, q_full, hh * 64, qrow);
              q_issued = true;
              return true;
            };
            auto independent = [&](int key0) { return !t.blk && key0 + 64 <= t.n; };
            if (!wprod) {  // Q region free once the previous unit's S MMAs are done
              const int r = mbar_wait_code(q_empty, ((uint32_t)qu & 1u) ^ 1u, a.status);
              if (r != 1) fwd_diag(a, r, 4, p, it, qu);
              if (r != 1 || (!independent(t.key_lo) && !issue_q())) {
                ok = false;
                break;
              }
            }
            for (int j = 0; j < t.tiles; ++j, ++it) {
              const int key0 = t.key_lo + j * 64;
              // Q before any wait that may need this unit's own S MMAs (a later tile's stage
              // can be one this unit's first tile frees)
              if (!wprod && (j >= 1 || !independent(key0)) && !q_issued && !issue_q()) {
                ok = false;
                break;
              }
              const int s = it % S;
              const uint32_t ph = (uint32_t)(it / S) & 1u;
              const int r = mbar_wait_code(&empty[s], ph ^ 1u, a.status);
              if (r != 1) {
                fwd_diag(a, r, wprod ? 1 : 2, p, it, s, 1);
                ok = false;
                break;
              }
              last_ph[s] = (int)ph;
              if (wprod) {
                mbar_arrive(&full[s]);  // attention tiles all come from the activation producer
                continue;
              }
              if (!independent(key0) && !dep_ready(dep)) {
                ok = false;
                break;
              }
              // K and V of the tile into one stage: K at 0, V at 128 d bytes (P follows them)
              uint8_t* st = stage_ptr(s);
              const CUtensorMap* mk = t.blk ? gm + G_KB64 : gm + G_KC64;
              const CUtensorMap* mv = t.blk ? gm + G_VB64 : gm + G_VC64;
              mbar_arrive_expect_tx(&full[s], 16384u * halves);
              for (int hh = 0; hh < halves; ++hh) tma_load_3d(st + hh * 8192, mk, &full[s], hh * 64, key0, zc);
              for (int hh = 0; hh < halves; ++hh)
                tma_load_3d(st + (halves + hh) * 8192, mv, &full[s], hh * 64, key0, zc);
            }
            if (ok && !wprod && !q_issued && !issue_q()) {
              ok = false;
              break;
            }
          }
        }
      }
      if (ok) {
        for (int s = 0; s < S; ++s)
          if (last_ph[s] >= 0) fwd_diag(a, mbar_wait_code(&full[s], (uint32_t)last_ph[s], a.status), 16, n_ph, it, s);
      }
      if (!ok || *(volatile int*)a.status != 0) {
        sleep_ns(20000);  // let loads already in flight land before the CTA can exit
        sleep_ns(20000);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t idesc_g = idesc_bf16(128, a.Mt, false);       // one activation plane (LM head)
      const uint32_t idesc_g2 = idesc_bf16(128, 2 * a.Mt, false);  // hi rows then lo rows
      const uint32_t idS = idesc_f16(128, 64, false);  // fp16 q and K
      const uint32_t idO = idesc_f16(128, d, true);    // fp16 P and V
      int it = 0, seg = 0, ta = 0, qu = 0;
      bool ok = true;
      for (int p = 0; ok && p < n_ph; ++p) {
        const int kind = fwd_phase_kind(p, a.L);
        if (!phase_active(g, kind)) continue;
        const int l = fwd_phase_layer(p);
        if (is_gemm_kind(kind)) {
          const GemmPhase gp = gemm_phase(a, kind, l);
          const long long W = gp.units;
          const long long u0 = unit_start(W, Gd, c), u1 = unit_start(W, Gd, c + 1);
          const int kc = gp.k_chunks;
          long long u = u0;
          while (ok && u < u1) {
            const int t = (int)(u / kc);
            const long long seg_start = u, seg_end = min(u1, (long long)(t + 1) * kc);
            const int buf = seg & 1, use = seg >> 1;
            int r = mbar_wait_code(&acce[buf], (uint32_t)(use & 1) ^ 1u, a.status);
            if (r != 1) {
              fwd_diag(a, r, 5, p, it, seg);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + buf * 256;
            for (; u < seg_end; ++u, ++it) {
              const int s = it % S;
              const uint32_t ph = (uint32_t)(it / S) & 1u;
              r = mbar_wait_code(&full[s], ph, a.status);
              if (r != 1) {
                fwd_diag(a, r, 6, p, it, s);
                ok = false;
                break;
              }
              if (u == u0) tl_mark<TL>(a, n_ph, p, TL_M0);
              tc_fence_after();
              const uint32_t wa = smem_u32(stage_ptr(s));
              const uint32_t xa = wa + 32768;
              // activation box [k chunk][plane][Mt][64]: per chunk, the B operand is the Mt hi rows
              // followed by the Mt lo rows, one MMA of N = 2 Mt (the weights are read once)
              const uint32_t x_chunk = (uint32_t)gp.planes * (uint32_t)a.Mt * 128u;
              const uint32_t idx = gp.planes == 2 ? idesc_g2 : idesc_g;
              // a descriptor's start address is (address >> 4) in its low 14 bits: an offset into
              // shared memory (below 256 KB) is added there directly
              const uint64_t wd0 = sw128_desc(wa, 16, 1024), xd0 = sw128_desc(xa, 16, 1024);
#pragma unroll
              for (int c2 = 0; c2 < 2; ++c2) {  // the two 64-wide k chunks of the unit
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ss(d_tmem, wd0 + (uint64_t)((c2 * 16384 + kk * 32) >> 4),
                         xd0 + (uint64_t)((c2 * x_chunk + kk * 32) >> 4), idx,
                         (u > seg_start || c2 > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit(&empty[s]);
            }
            if (!ok) break;
            mma_commit(&accf[buf]);
            ++seg;
          }
          if (u0 < u1) tl_mark<TL>(a, n_ph, p, TL_M1);
        } else if (kind == PH_ATTN) {
          const uint32_t qa = smem_u32(sQ);
          for (int u = c; ok && u < g.att_units; u += Gd, ++qu) {
            const AttUnit t = att_unit(a, g, lens_s, slot_pre, u);
            int r = mbar_wait_code(q_full, (uint32_t)qu & 1u, a.status);
            if (r != 1) {
              fwd_diag(a, r, 7, p, it, qu);
              ok = false;
              break;
            }
            // S = Q K^T of key tile jj (ring item itj, tile counter taj) into score buffer taj & 1
            auto issue_s = [&](int jj, int itj, int taj) -> bool {
              const int ks = itj % S;
              const int rr = mbar_wait_code(&full[ks], (uint32_t)(itj / S) & 1u, a.status);
              if (rr != 1) {
                fwd_diag(a, rr, 8, p, itj, ks);
                return false;
              }
              tc_fence_after();
              const uint64_t qd0 = sw128_desc(qa, 16, 1024), kd0 = sw128_desc(smem_u32(stage_ptr(ks)), 16, 1024);
              const uint32_t ts = (taj & 1) ? tS2 : tS;
#pragma unroll
              for (int kk = 0; kk < d / 16; ++kk)
                mma_ss(ts, qd0 + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                       kd0 + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), idS, kk > 0 ? 1u : 0u);
              mma_commit(&s_full[(taj & 1) * 3]);  // the stage is released after P V
              if (jj == t.tiles - 1) mma_commit(q_empty);  // last read of this unit's Q tile
              return true;
            };
            if (!issue_s(0, it, ta)) {
              ok = false;
              break;
            }
            for (int j = 0; ok && j < t.tiles; ++j, ++it, ++ta) {
              const int vs = it % S;  // this tile's stage (K, V and P); its full barrier was awaited for S
              // the next tile's scores go into the other buffer while the softmax warps work on
              // this one (its previous contents, tile j - 1, were read before P of j - 1)
              if (j + 1 < t.tiles && !issue_s(j + 1, it + 1, ta + 1)) {
                ok = false;
                break;
              }
              // P of this tile written (and O rescaled) by the softmax warps
              r = mbar_wait_code(&p_full[ta & 1], (uint32_t)(ta >> 1) & 1u, a.status);
              if (r != 1) {
                fwd_diag(a, r, 9, p, it, ta);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t va = smem_u32(stage_ptr(vs)) + (uint32_t)halves * 8192u, pa = va + (uint32_t)halves * 8192u;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tO, sw128_desc(pa + kk * 32, 16, 1024), sw128_desc(va + kk * 2048, 8192, 1024), idO,
                            (j > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&o_full[ta & 1]);
              mma_commit(&empty[vs]);
            }
            if (!ok) break;
          }
        }
      }
      mma_commit(done);
      mbar_wait(done, 0, a.status);
    }
  } else {
    // ======================= epilogue warps =======================
    fwd_epilogue_role<D_HEAD, TL, G2>(a, g, smem, stage_bytes, S, scr, red, rstd_s, lens_s, slot_pre, ust_s, accf, acce, full,
                              s_full, p_full, o_full, flag, tmem_base, tS, tO);
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(a.exit_cnt, 1);
    flag[7] = (old == Gd - 1) ? 1 : 0;
  }
  __syncthreads();
  if (flag[7]) {
    __threadfence();
    fwd_finalize(a, n_ph);
  }
}

}  // namespace orthrus
