// Internal launch interface between the context (pae_api.cu) and the kernel
// files.  Host-side declarations only.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace pae {

// Shapes the kernels need, fixed at pae_create.
struct Shape {
  int L, D, Hq, Hkv, d, F, A, H;
  int Bmax, Pmax, Ptot;  // Ptot = Pmax + H: slot length (prefix + action keys)
  int G;                 // Hq / Hkv
  int qkv_rows;          // (Hq + 2 Hkv) d
  int attn_dim;          // Hq d
  int group;             // W4A16 group size
  float eps;
  int table_rows;        // (2L*3 + 2) D floats per step
  int rope;              // 1: q and k heads are rotated (rows stored pair-interleaved)
  int Dp;                // prefix hidden width (0: no prefix production)
};

// Where the modulation of one norm sits inside a step's table row.
__host__ __device__ inline int mod_offset(const Shape& s, int layer, int norm, int chunk) {
  return ((layer * 2 + norm) * 3 + chunk) * s.D;
}
__host__ __device__ inline int final_offset(const Shape& s, int chunk) {
  return s.L * 2 * 3 * s.D + chunk * s.D;
}

// ------------------------------------------------------------ table builders
// t (device, K+1 doubles) -> e/c in `tc` [K][D] fp32 and dt [K].
void launch_time_mlp(const Shape& s, int act_bf16, const double* t, int K, const void* w_t1,
                     const void* b_t1, const void* w_t2, const void* b_t2, float* emb, float* zbuf,
                     float* cbuf, float* dt, cudaStream_t st);
// tables[k][r] = W_all[r] . c_k + b_all[r] for all table rows.
void launch_mod_tables(const Shape& s, int act_bf16, const float* cbuf, int K, const void* w_all,
                       const void* b_all, float* tables, cudaStream_t st);

// out[k][l][r] = W_l[r] . shift_k(l, norm) for every stored row r of the stacked
// bf16 matrix W ([L][rows][D]); out [K][L][rows] fp32.  norm 0 = attention,
// 1 = MLP adaRMSNorm.
void launch_shift_bias(const Shape& s, const void* W, int rows, int norm, const float* tables, int K, float* out,
                       cudaStream_t st);
// The same from packed int4 weights [L][rows][D/2] (create-time nibble order)
// and their group scales [L][rows][D/128].
void launch_shift_bias_w4(const Shape& s, const void* Wq, const void* scales, int rows, int norm,
                          const float* tables, int K, float* out, cudaStream_t st);

// ------------------------------------------------------------ token kernels
// Per token: optionally (final adaRMSNorm, out_proj, Euler update of x with
// step k_out), then optionally (in_proj of x and the first attention norm of
// step k_in).  Writes h (fp32) and y (act dtype).
struct TransitionArgs {
  float* x;               // [M][A]
  const float* x_src;     // read x from here in the first launch of a call (may equal x)
  float* h;               // [M][D]
  void* y;                // [M][D] act dtype
  const void* w_in; const void* b_in; const void* w_out; const void* b_out;
  const float* tab_out;   // table row of the step being finished (null: no out step)
  const float* dt;        // dt array (device)
  int k_out;
  const float* tab_in;    // table row of the step being started (null: no in step)
  float* x_dst;           // write x here after the out step (may equal x)
  int M;
  float* ss_out;          // non-null: the first norm's sum of squares per token -> ss_out[m] (slot 0)
  int y_factored;         // 1: y = bf16(h (1 + scale)) without rstd and shift (factored adaRMSNorm)
};
cudaError_t launch_transition(const Shape& s, int act_bf16, const TransitionArgs& a, bool pdl, cudaStream_t st);

// y = adaRMSNorm(h; scale, shift) per token.
cudaError_t launch_norm(const Shape& s, int act_bf16, const float* h, void* y, const float* scale,
                        const float* shift, int M, bool pdl, cudaStream_t st);

// Prefix production: y = h / sqrt(mean(h^2) + eps) per token, [len][Dp] act dtype.
cudaError_t launch_prefix_norm(int act_bf16, const void* h, void* y, int len, int Dp, float eps, cudaStream_t st);

// --------------------------------------------------------- CUDA-core (fp32)
enum Epi : int { EPI_QKV = 0, EPI_RESID = 1, EPI_GEGLU = 2, EPI_PREFIX = 3 };

struct EpiArgs {
  int epi;
  int M;
  // EPI_QKV
  void* q;            // [B][Hq][H][d] act dtype
  void* kc; void* vc; // [L][Bmax][Hkv][Ptot][d] act dtype
  const int* lens;    // [Bmax] prefix length per row
  int layer;
  // EPI_RESID
  float* h;           // [M][D]
  const float* gate;  // [D]
  float* ss_out;      // non-null: per-token sums of squares of the updated h, slot (tile * S + rank)
  int ss_ld;          // token stride of the sum-of-squares slots
  // EPI_GEGLU
  void* u;            // [M][F]
  // rotary embedding (EPI_QKV, EPI_PREFIX keys): (cos, sin) [Ptot][d/2], null = off
  const float2* rope_cs;
  // EPI_PREFIX: token m is prefix position m of request `prefix_row`; keys and
  // values go to kc / vc of `layer`
  int prefix_row;
  // Factored adaRMSNorm.  A consumer (EPI_QKV, EPI_GEGLU with f_ss set) reads
  // the operand bf16(h (1 + scale)) and applies out = rstd[m] acc + f_bias[row]
  // (f_bias: W shift of this step and layer, stored row order), rstd[m] =
  // rsqrt(sum of f_nslots slots (stride ss_ld) / D + eps).  The producer
  // (EPI_RESID with y_out set, split-K only) also writes y_out[m][f] =
  // bf16(h (1 + y_scale[f])) and the slots (ss_out).
  const float* f_bias;
  const float* f_ss;
  int f_nslots;
  void* y_out;
  const float* y_scale;
};

// out-features N (for GEGLU: F, weight rows interleaved in 128-row tiles).
void launch_gemm_simple(const Shape& s, const float* X, const float* W, int N, int K,
                        const EpiArgs& e, cudaStream_t st);

// o = attention(q, [prefix | action] keys) per request; CUDA cores.
void launch_attention_simple(const Shape& s, int act_bf16, const void* q, const void* kc,
                             const void* vc, const int* lens, int layer, void* o, int B,
                             cudaStream_t st);

// ----------------------------------------------------------- tcgen05 GEMM
struct TcPlan {
  int tn;          // token tile (MMA N), multiple of 16, <= 256
  int tok_tiles;
  int splits;      // split-K cluster size (power of two <= 16)
  int stages;
  int recv_alias;  // split-K receive buffer overlays the stage ring
};
struct TcGemmArgs {
  EpiArgs e;
  const bf16* scales;  // int4 weights: [rows][K/128] group scales (null: bf16 weights)
  // adaRMSNorm of the token operand inside the kernel (tmX is then the fp32
  // residual stream): rstd from nslots sum-of-squares slots, scale / shift rows
  const float* ss_in;
  int nslots, ss_ld;
  const float* nscale;
  const float* nshift;
  int N;           // output features (GEGLU: F)
  int K;
  int w_row0;      // first row of this layer's matrix inside the stacked weight map
  DevErr err;
};
cudaError_t launch_tc_gemm(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, int na,
                           const TcPlan& p, const TcGemmArgs& a, bool pdl, cudaStream_t st);
size_t tc_gemm_smem_bytes(int na, const TcPlan& p, bool w4, bool norm = false);
cudaError_t tc_gemm_init();  // once per process: opt in to large dynamic shared memory

// ------------------------------------------------------ tcgen05 attention
struct AttnPlan {
  int qtiles;          // ceil(G*H / 128) query tiles per (request, KV head)
  int splits;          // key splits (split-KV)
  int keys_per_split;  // multiple of 64 (and of chunk)
  int chunk;           // keys per attention chunk: 64 or 128
};
// Split-KV scratch: one slot per CTA of a split launch (the planner keeps
// those launches within one wave of 148 SMs), 128 rows each.
constexpr int kAttnMaxSplits = 8;
constexpr int kAttnPartSlots = 148;
struct AttnArgs {
  const int* lens;
  int layer;
  int keys_per_split;
  void* o;             // [M][Hq d] bf16, token-major
  __nv_bfloat16* part_o;  // [kAttnPartSlots][128][d] unnormalised partial rows (split-KV)
  float2* part_ml;        // [kAttnPartSlots][128] (row max, row sum) in the log2 domain
  DevErr err;
};
size_t attn_tc_smem_bytes(int d);
cudaError_t attn_tc_init();
cudaError_t launch_attn_tc(const Shape& s, const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                           const AttnPlan& p, const AttnArgs& a, int B, bool pdl, cudaStream_t st);

// ------------------------------------------- persistent loop (B*H <= 64)
// One projection of the persistent loop: nt tiles of 128 weight rows, each
// K range split over s CTAs (CTA i owns tile i / s, split i % s); na tiles
// form one reduction group (2: the gate and up tiles of the same features);
// reducer r of a group owns rows [r*rp, r*rp + rp).
struct PersistPhase {
  int nt, na, s, nkb, rp;
  int wrows;  // weight rows per layer in the stacked matrix
};
constexpr int kPersistGroups = 256;                     // counters per phase kind
constexpr int kPersistAbortIdx = 1 + 5 * kPersistGroups;  // launch-wide abort flag
constexpr int kPersistCtrWords = kPersistAbortIdx + 1;
struct PersistArgs {
  int M, ncta, k_begin, k_end;
  PersistPhase ph[4];  // QKV, O, gate/up, down
  int a_qtiles, a_splits, a_kps, a_items;
  float* x;
  float* h;
  bf16* q;
  bf16* o;
  bf16* u;
  bf16* kc;
  bf16* vc;
  const int* lens;
  const float* tables;
  const float* dt;
  const bf16* w_inT;
  const bf16* b_in;
  const bf16* w_out;
  const bf16* b_out;
  float* part;    // split-K / split-KV partials
  float* ss;      // [slot][64] per-token sums of squares of the residual stream
  unsigned* ctr;  // [kPersistCtrWords], zero at launch
  DevErr err;
};
size_t persist_smem_bytes();
cudaError_t persist_init();
// Cooperative launch of a.ncta CTAs (one per SM).
cudaError_t launch_persistent(const Shape& s, const CUtensorMap* maps /* Wqkv, Wo, Wgu (128-row box), Wdown, Q, K, V */,
                              const PersistArgs& a, cudaStream_t st);

// ------------------------------------ dataflow loop (B*H <= 64, clusters)
// One launch of NC clusters of C CTAs runs all Euler steps of a call; stages
// wait on per-tile counters (k_flow.cu).
constexpr int kFlowCtrWords = 512;  // counters; the last word is the abort flag
struct FlowArgs {
  int M, B;                          // tokens, requests
  int C, NC;                         // cluster size, clusters
  int k_begin, k_end;                // Euler steps of this launch
  int q_units, o_tiles, g_units, d_tiles;  // QKV / gate-up whole-K units, O / down split-K tiles (128 rows)
  int q_base, o_base, g_base, d_base, a_base;  // first CTA (units) or cluster (tiles, attention)
  int kb_q, kb_o, kb_g, kb_d;        // 64-wide K blocks per unit (QKV, gate/up) or per rank (O, down)
  int a_units, a_qtiles, a_kps;      // attention clusters, query tiles per (b, kv head), keys per rank
  float* x;
  float* h;
  bf16* yq;                          // bf16(h (1 + scale)) of the attention norm [64][D]
  bf16* yg;                          // the same for the MLP norm
  bf16* q;
  bf16* o;
  bf16* u;
  bf16* kc;
  bf16* vc;
  const int* lens;
  const float* tables;
  const float* dt;
  const float* bias_qkv;             // [K][L][qkv_rows]  W_qkv shift_attention
  const float* bias_gu;              // [K][L][2F]        W_gate/up shift_mlp (stored row order)
  float* ss_q;                       // [d_tiles * C][64] sums of squares for the QKV norm
  float* ss_g;                       // [o_tiles * C][64] for the MLP norm
  float* ss_t;                       // [64] from the transition (layer 0)
  const bf16* w_inT;
  const bf16* b_in;
  const bf16* w_out;
  const bf16* b_out;
  const float2* rope_cs;
  int w4;                            // int4 weights (packed maps; wsc = group scales)
  const bf16* wsc[4];                // W4A16: [rows][K/128] scales of QKV, O, gate/up (stored order), down
  unsigned* ctr;                     // [kFlowCtrWords], zero at launch
  DevErr err;
};
size_t flow_smem_bytes();
cudaError_t flow_init();
int flow_max_clusters(int C);        // clusters of C CTAs that fit at once (0 on error)
// maps: W qkv, W o, W gate/up (64-row boxes), W down (bf16 [128][64] boxes,
// gate/up [64][64]; with w4 the packed [128 rows][32 bytes] boxes, gate/up
// [64][32 bytes]), y_q, o, y_g, u (64 x 64 boxes), q (64 x 128), k, v
// (64 x 64).  Cooperative cluster launch.
cudaError_t launch_flow(const Shape& s, const CUtensorMap* maps, const FlowArgs& a, cudaStream_t st);

}  // namespace pae
