// The C ABI of include/pae.h: context lifetime, weight repacking, prefix slots,
// timestep tables, and the K-step loop (enqueued directly or replayed from a
// captured CUDA graph).
//
// The loop structure is the pi0.5 path of "PhyAI: Real-Time Physical AI at
// the Edge" (Sec. 5.1 and Sec. 5.5): the prefix K/V stays fixed across the
// Euler steps and is replaced only by a new observation (pae_set_prefix), the
// timestep/modulation tables are built once (pae_precompute_tables), and the
// stable loop is replayed as a CUDA graph (pae_denoise).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "pae.h"
#include "internal.h"
#include "epilogue.cuh"

using namespace pae;

namespace {

thread_local std::string g_create_error;

}  // namespace

namespace pae {
// Message that pae_last_error(NULL) reports (context-free entry points).
void set_create_error(const char* msg) { g_create_error = msg ? msg : ""; }
}  // namespace pae

namespace {

constexpr int kMaxSteps = 64;
constexpr int kSsSlots = 256;  // sum-of-squares slots: (D / 128) tiles x split-K ranks
constexpr int kDefaultMaxSplitK = 8;  // PAE_OPT_MAX_SPLITK until set

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct ProfRec {
  int kind;
  int ev0, ev1;  // indices into the context's event pool
};

struct Plan {
  int B = 0, M = 0;
  TcPlan qkv{}, o{}, gu{}, down{};
  AttnPlan attn{};
  bool persist = false;  // eligible for the persistent kernel
  PersistArgs pa{};
  bool flow = false;       // eligible for the dataflow loop (clusters, per-tile counters)
  FlowArgs fa{};
  bool fuse_norm = false;  // QKV / gate-up normalise their fp32 operand in-kernel
  bool factored = false;   // adaRMSNorm factored into the projections' epilogues (no norm kernels)
  // token-operand maps; a map's box height is the token tile of the projection
  // that reads it (QKV and gate/up may tile the same y differently)
  CUtensorMap tmY{}, tmYg{}, tmO{}, tmU{}, tmH{}, tmHg{};
  cudaGraphExec_t graph = nullptr;
  int graph_K = 0;
  long long graph_kernels = 0;
  std::vector<ProfRec> recs;  // profiled launches of the last enqueue / capture
};

__global__ void k_set_len(int* lens, int row, int len) { lens[row] = len; }

template <typename T>
__global__ void k_transpose(const T* __restrict__ src, T* __restrict__ dst, int rows, int cols) {
  // dst[c][r] = src[r][c]
  const size_t n = (size_t)rows * cols;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / cols, c = i - r * cols;
    dst[c * rows + r] = src[i];
  }
}

// Rotary pairing of the q/k block (rows [0, rot_rows), head_dim d): stored row
// p of a head holds channel rope_channel(p) = p/2 + (p odd) d/2, so the two
// channels a rotation mixes leave the GEMM side by side.  dst[r] = src[src_row(r)]
// in units of 2 bytes, `cols` units per row; rows past rot_rows are copied as is.
__global__ void k_permute_rows(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int rows, int cols,
                               int rot_rows, int d) {
  const size_t n = (size_t)rows * cols;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), c = (int)(i - (size_t)r * cols);
    const int sr = r < rot_rows ? (r / d) * d + rope_channel(r % d, d) : r;
    dst[i] = src[(size_t)sr * cols + c];
  }
}

// Packed int4 rows [rows][kbytes] -> the kernels' layout: within every
// 32-bit word the nibbles of k = 0..7 move to bit positions
// 0, 16, 4, 20, 8, 24, 12, 28, so that (w >> 4i) & 0x000F000F holds the
// pair (k = 2i, 2i + 1).  Row r goes to destination row dst_row(r):
// mode 0 identity, 1 gate rows and 2 up rows of the 128-row interleave.
__global__ void k_repack_int4(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int rows, int kbytes,
                              int mode, int rot_rows, int d) {
  const int words = kbytes / 4;
  const size_t n = (size_t)rows * words;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / words), c = (int)(i - (size_t)r * words);
    const uint32_t w = reinterpret_cast<const uint32_t*>(src + (size_t)r * kbytes)[c];
    uint32_t o = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t nib = (w >> (4 * k)) & 0xFu;
      const int pos = (k & 1) ? 16 + 4 * (k >> 1) : 4 * (k >> 1);
      o |= nib << pos;
    }
    // mode 0 with rotation: source channel j of a q/k head goes to stored row
    // 2j (j < d/2) or 2(j - d/2) + 1
    int dr = mode == 0 ? r : ((r >> 7) * 256 + (r & 127) + (mode == 2 ? 128 : 0));
    if (mode == 0 && r < rot_rows) {
      const int j = r % d, h2 = d >> 1;
      dr = (r / d) * d + (j < h2 ? 2 * j : 2 * (j - h2) + 1);
    }
    reinterpret_cast<uint32_t*>(dst + (size_t)dr * kbytes)[c] = o;
  }
}

}  // namespace

struct pae_ctx {
  pae_config cfg{};
  Shape s{};
  int device = 0;
  int act_bf16 = 0;  // bf16 activations (BF16 and W4A16 modes)
  size_t esize = 4;  // bytes per weight element (non-quantised)
  std::vector<void*> allocs;
  // weights (device, repacked)
  void *w_inT = nullptr, *b_in = nullptr, *w_out = nullptr, *b_out = nullptr;
  void *w_t1 = nullptr, *b_t1 = nullptr, *w_t2 = nullptr, *b_t2 = nullptr;
  void *w_modall = nullptr, *b_modall = nullptr;
  void *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_down = nullptr;  // stacked over layers
  CUtensorMap tmWqkv{}, tmWo{}, tmWgu{}, tmWdown{};
  CUtensorMap tmQ{}, tmK{}, tmV{};  // attention operands (bf16 modes), 64-key boxes
  CUtensorMap tmWgu1{};             // gate/up weights with 128-row boxes (persistent kernel)
  // persistent kernel: one CTA per SM, split-K / split-KV workspace, counters
  int ncta = 0;
  bool use_persistent = false;  // opt-in: measured slower than the graph at batch 1
  float* pw_part = nullptr;
  float* pw_ss = nullptr;
  unsigned* pw_ctr = nullptr;
  // dataflow loop (batch * chunk <= 64): the MLP norm's operand, sums of
  // squares, the projected adaRMSNorm shifts per step, counters, 64-row maps
  bool flow_capable = false;
  bool use_flow = false;  // opt-in until it beats the captured graph at batch 1
  int flow_cluster = 0;          // 0: automatic
  int flow_max_cl[17] = {};      // clusters of C CTAs that fit at once
  void* yg = nullptr;
  float *f_ssq = nullptr, *f_ssg = nullptr, *f_sst = nullptr;
  float *bias_qkv = nullptr, *bias_gu = nullptr;
  unsigned* f_ctr = nullptr;
  CUtensorMap tmYq64{}, tmYg64{}, tmO64{}, tmU64{};
  CUtensorMap tmWg64{};  // gate/up with 64-row boxes (dataflow loop)
  // in-kernel adaRMSNorm: per-token sum-of-squares slots [kSsSlots][ss_ld]
  bool use_fused_norm = false;  // opt-in: measured slower than the norm kernels under PDL
  bool use_factored = false;    // opt-in: measured slower than the norm kernels under PDL
  float* ss_buf = nullptr;
  int ss_ld = 0;
  // split-KV merge scratch: partial rows [kAttnPartSlots][128][d] bf16, then (max, sum) [kAttnPartSlots][128]
  void* attn_part = nullptr;
  // int4 weights (W4A16): packed codes [L*rows][K/2] and group scales [L*rows][K/128]
  int w4 = 0;
  void *q_qkv = nullptr, *q_o = nullptr, *q_gu = nullptr, *q_down = nullptr;
  void *sc_qkv = nullptr, *sc_o = nullptr, *sc_gu = nullptr, *sc_down = nullptr;
  CUtensorMap tmQqkv{}, tmQo{}, tmQgu{}, tmQdown{};
  CUtensorMap tmQg64{};  // packed gate/up with 64-row boxes (dataflow loop)
  // tables
  double* t_dev = nullptr;
  float *emb = nullptr, *zbuf = nullptr, *cbuf = nullptr, *tables = nullptr, *dt = nullptr;
  int K = 0;
  bool tables_ready = false;
  // rotary embedding: (cos, sin) of position x channel pair, [Ptot][d/2]
  float2* rope_cs = nullptr;
  // prefix production: key/value rows per layer [L][2 Hkv d][Dp] (keys paired
  // like the q/k block when rotating) and the normalised hidden states [Pmax][Dp]
  void* w_pkv = nullptr;
  void* ypre = nullptr;
  CUtensorMap tmWpkv{}, tmYpre{};
  // prefix slots
  void *kc = nullptr, *vc = nullptr;
  int* lens_dev = nullptr;
  std::vector<int> lens_host;
  // activations and workspaces
  float *x = nullptr, *h = nullptr;
  void *y = nullptr, *q = nullptr, *o = nullptr, *u = nullptr;
  // error word (host-mapped)
  int* err_host = nullptr;
  int* err_dev = nullptr;
  long long wait_ns = 2000000000LL;
  bool use_graph = true;
  bool use_pdl = true;
  int max_splitk = kDefaultMaxSplitK;
  std::map<int, Plan> plans;
  Plan* last_plan = nullptr;
  unsigned profile_mask = 0;
  std::vector<cudaEvent_t> ev_pool;
  int ev_next = 0;
  std::vector<ProfRec>* rec_sink = nullptr;
  // First error a launch helper returned while enqueue_steps ran: one that
  // rejects its arguments returns before launching, so the runtime's last
  // error would not show it.
  cudaError_t enq_err = cudaSuccess;
  cudaStream_t cap_stream = nullptr;
  EncodeTiledFn encode = nullptr;
  std::string last_error;
};

namespace {

pae_status fail(pae_ctx* c, pae_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (c)
    c->last_error = buf;
  else
    g_create_error = buf;
  return st;
}

#define CK(call)                                                                              \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) return fail(ctx, PAE_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

pae_status dev_alloc(pae_ctx* ctx, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ctx, PAE_ERR_OOM, "cudaMalloc(%zu bytes): %s", bytes, cudaGetErrorString(e));
  }
  ctx->allocs.push_back(*p);
  return PAE_OK;
}

pae_status check_err_word(pae_ctx* ctx) {
  if (ctx->err_host && *(volatile int*)ctx->err_host != 0) {
    const int code = *(volatile int*)ctx->err_host;
    if (code == DEV_DRAIN)
      return fail(ctx, PAE_ERR_TIMEOUT, "device error word set (%d): a drain of copies or MMAs already issued ran "
                                        "out; destroy this context", code);
    return fail(ctx, PAE_ERR_TIMEOUT, "device error word set (%d): a bounded device wait ran out", code);
  }
  return PAE_OK;
}

pae_status make_map(pae_ctx* ctx, CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint32_t box_inner, uint32_t box_outer) {
  // bf16 matrix [outer][inner], 128-byte swizzled boxes of box_inner x box_outer.
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, PAE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%llu][%llu] box %ux%u", (int)r,
                (unsigned long long)outer, (unsigned long long)inner, box_outer, box_inner);
  return PAE_OK;
}

pae_status make_map_f32(pae_ctx* ctx, CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                        uint32_t box_inner, uint32_t box_outer) {
  // fp32 matrix [outer][inner], unswizzled boxes (the residual stream tiles).
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, PAE_ERR_CUDA, "cuTensorMapEncodeTiled (fp32) failed (%d)", (int)r);
  return PAE_OK;
}

pae_status make_map_u8(pae_ctx* ctx, CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer) {
  // uint8 matrix [outer][inner], unswizzled boxes (the packed int4 tiles).
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, PAE_ERR_CUDA, "cuTensorMapEncodeTiled (uint8) failed (%d)", (int)r);
  return PAE_OK;
}

// Token tile and split-K choice for one projection of `nfeat` outputs and K
// inputs.  The token tile covers the tokens with as little padding as possible
// (<= 256 per MMA).  Split-K (a cluster of S CTAs, S a power of two <= 16 that
// divides the 64-wide K blocks) fills the 148 SMs when the tile count is small;
// small token tiles keep shared memory under half an SM so that two CTAs (or a
// CTA and its successor under PDL) fit per SM.
// Ring depth and receive-buffer placement for a token tile / split choice
// within a shared-memory budget (false if fewer than two stages fit).  A
// separate split-K receive buffer saves a cluster barrier, but it is taken
// only when it costs no ring depth: on long K loops a shallow ring starves the
// tensor cores (measured on the batch-32 down projection).
bool fit_ring(TcPlan& p, int na, int nkb, bool w4, bool norm, uint32_t budget) {
  const uint32_t stage = (uint32_t)na * 16384u + (uint32_t)p.tn * 128u + (w4 ? (uint32_t)na * 4096u : 0u) +
                         (norm ? (uint32_t)p.tn * 128u : 0u);
  const uint32_t recv = p.splits > 1 ? (uint32_t)na * p.tn * 128u * 4u : 0u;
  int st = std::min((int)(budget / stage), 8);
  st = std::min(st, std::max(2, nkb / p.splits));
  if (st < 2) return false;
  p.recv_alias = 0;
  if (p.splits > 1) {
    const int st_sep = std::min(st, (int)((budget - std::min(budget, recv)) / stage));
    if (st_sep >= st) {
      st = st_sep;
    } else {
      p.recv_alias = 1;
      st = std::max(st, (int)((recv + stage - 1) / stage));
    }
  }
  p.stages = st;
  return true;
}

// Large batches (more than one 256-token tile): one CTA per SM (token tiles of
// 128..256 need most of the shared memory), so choose the token-tile count
// whose CTAs (output tiles x split-K, split-K as long as the tiles fit one
// wave) fill whole waves of 148 SMs best; ties go to the larger tile.  At
// M = 1600 this picks 240 for QKV (140 CTAs), 192 with split-K 2 for O and
// down (144) and 192 for gate/up (288 = two full waves), which measured
// 23.4 ms per batch-32 call against 24.7 ms for a fixed 240-token tile.
TcPlan plan_gemm_large(int M, int nfeat, int K, int na, int max_splits, bool w4, bool norm) {
  const int nt = (nfeat + 127) / 128, nkb = K / 64;
  TcPlan best{};
  double best_eff = -1.0;
  for (int tt = (M + 255) / 256; tt <= (M + 127) / 128; ++tt) {
    const int tn = (((M + tt - 1) / tt + 15) / 16) * 16;
    if (tn > 256 || tn < 128 || (M + tn - 1) / tn != tt) continue;
    const int base = nt * tt;
    int sp = 1;
    for (int c = 2; c <= std::min(8, max_splits); c *= 2)
      if (nkb % c == 0 && base * c <= 148) sp = c;
    TcPlan p{};
    p.tn = tn;
    p.tok_tiles = tt;
    p.splits = sp;
    if (!fit_ring(p, na, nkb, w4, norm, 200u * 1024u)) continue;
    const int ctas = base * sp;
    const int waves = (ctas + 147) / 148;
    const double eff = (double)ctas / (148.0 * waves);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = p;
    }
  }
  return best;
}

// whole_sm (small batches): the projection follows the norm kernel, which
// holds no shared memory, so its CTAs can take a whole SM and still start
// early under programmatic dependent launch: split-K only as far as one CTA
// per SM (tiles x splits <= 148) with a deep ring.  Measured at batch 1
// (QKV 20 tiles -> split 4, gate/up 32 tiles -> split 4): 9.0 ms per call
// against 9.6 ms with split 8 and two CTAs per SM (int4 weights: 9.5 against
// 10.5 ms).  O and down follow the
// attention and gate/up kernels, which fill most of an SM's shared memory, and
// keep the two-CTA footprint (splitting them 4 or 16 ways measured slower).
TcPlan plan_gemm(int M, int nfeat, int K, int na, int max_splits = 16, bool w4 = false, bool norm = false,
                 bool whole_sm = false) {
  if (M > 256) {
    const TcPlan p = plan_gemm_large(M, nfeat, K, na, max_splits, w4, norm);
    if (p.tn > 0) return p;
  }
  TcPlan p{};
  p.tok_tiles = (M + 255) / 256;
  int per = (M + p.tok_tiles - 1) / p.tok_tiles;
  p.tn = std::max(16, ((per + 15) / 16) * 16);
  const int base = ((nfeat + 127) / 128) * p.tok_tiles;
  const int nkb = K / 64;
  const uint32_t stage = (uint32_t)na * 16384u + (uint32_t)p.tn * 128u + (w4 ? (uint32_t)na * 4096u : 0u) +
                         (norm ? (uint32_t)p.tn * 128u : 0u);
  const uint32_t recv = (uint32_t)na * p.tn * 128u * 4u;  // split-K receive buffer
  // two CTAs per SM (shared memory and the 128-register cap allow it)
  const bool small = p.tn <= 64 && !whole_sm;
  const uint32_t budget = small ? 110u * 1024u : 200u * 1024u;
  const int target = small ? 2 * 148 : 148;
  p.splits = 1;
  for (int sp = 2; sp <= std::min(16, max_splits); sp *= 2)
    if (nkb % sp == 0 && base * sp <= target && recv <= budget) p.splits = sp;
  if (whole_sm && p.tn <= 64 && fit_ring(p, na, nkb, w4, norm, budget)) return p;
  // without split-K a CTA streams a long K range: give it a deep ring
  const uint32_t ring_budget = p.splits == 1 ? 200u * 1024u : budget;
  int st = std::max(2, std::min((int)(ring_budget / stage), 8));
  st = std::min(st, std::max(2, nkb / p.splits));
  p.recv_alias = 0;
  if (p.splits > 1) {
    // a separate receive buffer saves a cluster barrier; overlay it on the
    // ring when both do not fit
    int st_sep = std::min(st, (int)((budget - std::min(budget, recv)) / stage));
    if (st_sep >= 2) {
      st = st_sep;
    } else {
      p.recv_alias = 1;
      st = std::max(st, (int)((recv + stage - 1) / stage));
    }
  }
  p.stages = st;
  return p;
}

// Query tiles of 128 rows per (request, KV head); key splits (a cluster of
// S <= 8 CTAs, S a power of two) only when the batch gives too few tiles to
// fill the 148 SMs (split-KV at small batch).
AttnPlan plan_attn(const Shape& s, int B) {
  AttnPlan p{};
  p.qtiles = (s.G * s.H + 127) / 128;
  const int base = B * s.Hkv * p.qtiles;
  const int max_splits = (s.Ptot + 63) / 64;
  int splits = 1;
  // at most 8: 16 splits (one 64-key chunk per CTA at batch 1) measured
  // slower, 21.2 against 19.7 us per launch (the merge grows with the ranks)
  while (splits < 8 && base * splits * 2 <= 148 && splits * 2 <= max_splits) splits *= 2;
  p.keys_per_split = ((s.Ptot + splits - 1) / splits + 63) / 64 * 64;
  p.splits = splits;
  // 128-key chunks (half the softmax passes, S with N = 128) for key ranges of
  // two or more such chunks (the split rounded up to whole chunks): batch 32,
  // 20.7 -> 20.0-20.3 ms per call.  A split of 128 keys keeps two 64-key
  // chunks, whose softmax and PV overlap (one 128-key chunk measured 8.79
  // against 8.76 ms per batch-1 call).
  p.chunk = 64;
  if (p.keys_per_split >= 256) {
    p.keys_per_split = (p.keys_per_split + 127) / 128 * 128;
    p.chunk = 128;
  }
  return p;
}

// Persistent-kernel plan for M = B*H <= 64 tokens (bf16 weights): every
// projection's K range is split so that its tiles x splits fill the SMs; the
// attention keys are split into 64-key chunks over the (request, KV head,
// query tile) groups.  Returns false when the batch or shape is not eligible.
bool plan_persistent(const pae_ctx* ctx, int B, PersistArgs* pa) {
  const Shape& s = ctx->s;
  const int M = B * s.H, n = ctx->ncta;
  if (!ctx->act_bf16 || ctx->w4 || s.rope || n < 1 || M > 64 || M > n) return false;
  if (s.d != 64 && s.d != 128 && s.d != 256) return false;
  if ((size_t)(s.D + s.A) * 4 > 128 * 1024) return false;
  *pa = PersistArgs{};
  pa->M = M;
  pa->ncta = n;
  auto mk = [&](PersistPhase& p, int rows, int K, int na, bool resid) -> bool {
    p.nt = rows / 128;
    p.na = na;
    p.nkb = K / 64;
    p.wrows = rows;
    if (p.nt < 1 || p.nt > n || p.nt / na > kPersistGroups) return false;
    p.s = std::max(1, std::min(n / p.nt, p.nkb));
    if ((p.nkb + p.s - 1) / p.s > 16) return false;  // token operand must fit the 128 KB work area
    int q4 = ((128 + na * p.s - 1) / (na * p.s) + 3) / 4;
    if (resid) {
      int pw = 1;
      while (pw < q4) pw <<= 1;
      q4 = pw;
    }
    p.rp = 4 * q4;
    return true;
  };
  if (!mk(pa->ph[0], s.qkv_rows, s.D, 1, false) || !mk(pa->ph[1], s.D, s.attn_dim, 1, true) ||
      !mk(pa->ph[2], 2 * s.F, s.D, 2, false) || !mk(pa->ph[3], s.D, s.F, 1, true))
    return false;
  pa->a_qtiles = (s.G * s.H + 127) / 128;
  const int base = B * s.Hkv * pa->a_qtiles;
  if (base > n || base > kPersistGroups) return false;
  const int chunks = (s.Ptot + 63) / 64;
  int sa = std::max(1, std::min(chunks, n / base));
  pa->a_kps = 64 * ((chunks + sa - 1) / sa);
  sa = (s.Ptot + pa->a_kps - 1) / pa->a_kps;
  pa->a_splits = sa;
  pa->a_items = base * sa;
  pa->x = ctx->x;
  pa->h = ctx->h;
  pa->q = static_cast<bf16*>(ctx->q);
  pa->o = static_cast<bf16*>(ctx->o);
  pa->u = static_cast<bf16*>(ctx->u);
  pa->kc = static_cast<bf16*>(ctx->kc);
  pa->vc = static_cast<bf16*>(ctx->vc);
  pa->lens = ctx->lens_dev;
  pa->tables = ctx->tables;
  pa->dt = ctx->dt;
  pa->w_inT = static_cast<const bf16*>(ctx->w_inT);
  pa->b_in = static_cast<const bf16*>(ctx->b_in);
  pa->w_out = static_cast<const bf16*>(ctx->w_out);
  pa->b_out = static_cast<const bf16*>(ctx->b_out);
  pa->part = ctx->pw_part;
  pa->ss = ctx->pw_ss;
  pa->ctr = ctx->pw_ctr;
  return true;
}

// Dataflow-loop plan for M = B*H <= 64 tokens.  QKV and gate/up run as
// 128-row whole-K units, one CTA each (the token operand, 64 x width bf16,
// within the 128 KB work area: width <= 1024); at most 8 units per CTA (TMEM
// columns).  O and down split K over the C ranks of a cluster with a
// 64-wide block count per rank and the operand slice within 64 KB.  The grid
// is as many clusters of C as fit at once (one CTA per SM), which must cover
// the attention units (request, KV head, 128 query rows) and the M token CTAs
// of the transition.  Preferred: every O and down tile on a cluster of its
// own, then the larger C (fewer K blocks per rank).  Returns false when the
// batch or shape is not eligible.
bool plan_flow(const pae_ctx* ctx, int B, FlowArgs* fa) {
  const Shape& s = ctx->s;
  const int M = B * s.H;
  if (!ctx->flow_capable || M < 1 || M > 64) return false;
  if (s.D % 128 || s.D > 1024 || s.qkv_rows % 128 || s.F % 128 || s.attn_dim % 64) return false;
  const int nkD = s.D / 64, nkA = s.attn_dim / 64, nkF = s.F / 64;
  const int qtiles = (s.G * s.H + 127) / 128;
  const int units = B * s.Hkv * qtiles;
  const int q_units = s.qkv_rows / 128, g_units = s.F / 64, tiles = s.D / 128;
  if (3 + 2 * tiles + g_units + 1 > kFlowCtrWords) return false;
  if (s.d > 256 || 128 * s.d * 2 + 2 * 64 * s.d * 2 > 128 * 1024) return false;
  int bestC = 0, bestNC = 0;
  bool bestFit = false;
  for (int C : {16, 8, 4, 2}) {
    if (ctx->flow_cluster && C != ctx->flow_cluster) continue;
    if (nkA % C || nkF % C) continue;
    if ((nkF / C) * 8192 > 64 * 1024 || (nkA / C) * 8192 > 64 * 1024) continue;
    const int NC = std::min(ctx->flow_max_cl[C], 148 / C), ncta = NC * C;
    if (NC < 1 || NC < units || ncta < M) continue;
    if ((q_units + ncta - 1) / ncta > 8 || (g_units + ncta - 1) / ncta > 8) continue;
    const bool fit = tiles <= NC;
    if (!bestC || (fit && !bestFit)) {
      bestC = C;
      bestNC = NC;
      bestFit = fit;
    }
  }
  if (!bestC) return false;
  *fa = FlowArgs{};
  fa->M = M;
  fa->B = B;
  fa->C = bestC;
  fa->NC = bestNC;
  fa->q_units = q_units;
  fa->o_tiles = tiles;
  fa->g_units = g_units;
  fa->d_tiles = tiles;
  // O tiles from cluster 0, down tiles on the last clusters, attention after
  // the O tiles; QKV units from CTA 0, gate/up units after them
  fa->o_base = 0;
  fa->d_base = std::max(0, bestNC - tiles);
  fa->a_base = tiles < bestNC ? tiles : 0;
  fa->q_base = 0;
  fa->g_base = q_units % (bestNC * bestC);
  fa->kb_q = nkD;
  fa->kb_o = nkA / bestC;
  fa->kb_g = nkD;
  fa->kb_d = nkF / bestC;
  fa->a_units = units;
  fa->a_qtiles = qtiles;
  const int chunks = (s.Ptot + 63) / 64;
  fa->a_kps = 64 * ((chunks + bestC - 1) / bestC);
  fa->x = ctx->x;
  fa->h = ctx->h;
  fa->yq = static_cast<bf16*>(ctx->y);
  fa->yg = static_cast<bf16*>(ctx->yg);
  fa->q = static_cast<bf16*>(ctx->q);
  fa->o = static_cast<bf16*>(ctx->o);
  fa->u = static_cast<bf16*>(ctx->u);
  fa->kc = static_cast<bf16*>(ctx->kc);
  fa->vc = static_cast<bf16*>(ctx->vc);
  fa->lens = ctx->lens_dev;
  fa->tables = ctx->tables;
  fa->dt = ctx->dt;
  fa->bias_qkv = ctx->bias_qkv;
  fa->bias_gu = ctx->bias_gu;
  fa->ss_q = ctx->f_ssq;
  fa->ss_g = ctx->f_ssg;
  fa->ss_t = ctx->f_sst;
  fa->w_inT = static_cast<const bf16*>(ctx->w_inT);
  fa->b_in = static_cast<const bf16*>(ctx->b_in);
  fa->w_out = static_cast<const bf16*>(ctx->w_out);
  fa->b_out = static_cast<const bf16*>(ctx->b_out);
  fa->rope_cs = ctx->rope_cs;
  fa->w4 = ctx->w4;
  fa->wsc[0] = static_cast<const bf16*>(ctx->sc_qkv);
  fa->wsc[1] = static_cast<const bf16*>(ctx->sc_o);
  fa->wsc[2] = static_cast<const bf16*>(ctx->sc_gu);
  fa->wsc[3] = static_cast<const bf16*>(ctx->sc_down);
  fa->ctr = ctx->f_ctr;
  return true;
}

// The launch shapes of one batch size (tensor-core modes): host arithmetic
// only, shared by the context and pae_plan_query.
struct LaunchPlans {
  TcPlan qkv, o, gu, down;
  AttnPlan attn;
  bool fuse_norm;
  bool factored;
};
LaunchPlans plan_launches(const Shape& s, int B, bool w4, int max_splitk, bool use_fused_norm,
                          bool use_factored) {
  LaunchPlans L{};
  const int M = B * s.H;
  L.o = plan_gemm(M, s.D, s.attn_dim, 1, max_splitk, w4);
  L.down = plan_gemm(M, s.D, s.F, 1, max_splitk, w4);
  // In-kernel adaRMSNorm for small batches (one token tile of <= 64): the
  // residual projections' split-K ranks (R = 128 / S <= 32 rows each) write
  // the sum-of-squares slots, so the separate norm kernels disappear.
  const int tn_small = std::max(16, ((M + 15) / 16) * 16);
  L.fuse_norm = use_fused_norm && !w4 && M <= 64 && tn_small <= 64 && L.o.splits >= 4 && L.down.splits >= 4 &&
                L.o.tok_tiles == 1 && L.down.tok_tiles == 1 &&
                (s.D / 128) * std::max(L.o.splits, L.down.splits) <= kSsSlots;
  // Factored adaRMSNorm: the residual projections' split-K epilogue writes
  // the next operand bf16(h (1 + scale)) and per-token sums of squares (one
  // slot per tile and rank), and QKV / gate-up apply rstd and the projected
  // shift in their epilogues: no norm kernels.
  L.factored = use_factored && !L.fuse_norm && L.o.splits >= 2 && L.down.splits >= 2 &&
               (s.D / 128) * std::max(L.o.splits, L.down.splits) <= kSsSlots;
  // QKV and gate/up take a whole SM only after a norm kernel, which holds no
  // shared memory; after a projection they keep the two-CTA footprint so
  // that they can start beside its last CTAs.
  const bool whole_sm = !L.fuse_norm && !L.factored;
  L.qkv = plan_gemm(M, s.qkv_rows, s.D, 1, max_splitk, w4, L.fuse_norm, whole_sm);
  L.gu = plan_gemm(M, s.F, s.D, 2, max_splitk, w4, L.fuse_norm, whole_sm);
  L.attn = plan_attn(s, B);
  return L;
}

pae_status build_plan(pae_ctx* ctx, int B, Plan* P) {
  const Shape& s = ctx->s;
  P->B = B;
  P->M = B * s.H;
  if (!ctx->act_bf16) return PAE_OK;
  P->persist = plan_persistent(ctx, B, &P->pa);
  P->flow = plan_flow(ctx, B, &P->fa);
  const LaunchPlans LP = plan_launches(s, B, ctx->w4 != 0, ctx->max_splitk, ctx->use_fused_norm, ctx->use_factored);
  P->qkv = LP.qkv;
  P->o = LP.o;
  P->gu = LP.gu;
  P->down = LP.down;
  P->attn = LP.attn;
  if (P->attn.splits > 1 &&
      (P->attn.splits > kAttnMaxSplits || B * s.Hkv * P->attn.qtiles * P->attn.splits > kAttnPartSlots))
    return fail(ctx, PAE_ERR_UNSUPPORTED, "split-KV plan exceeds the merge scratch (%d splits)", P->attn.splits);
  P->fuse_norm = LP.fuse_norm;
  P->factored = LP.factored;
  const uint64_t Mmax = (uint64_t)s.Bmax * s.H;
  pae_status st;
  if ((st = make_map(ctx, &P->tmY, ctx->y, s.D, Mmax, 64, P->qkv.tn)) != PAE_OK) return st;
  if ((st = make_map(ctx, &P->tmYg, ctx->y, s.D, Mmax, 64, P->gu.tn)) != PAE_OK) return st;
  if ((st = make_map(ctx, &P->tmO, ctx->o, s.attn_dim, Mmax, 64, P->o.tn)) != PAE_OK) return st;
  if ((st = make_map(ctx, &P->tmU, ctx->u, s.F, Mmax, 64, P->down.tn)) != PAE_OK) return st;
  if (P->fuse_norm && (st = make_map_f32(ctx, &P->tmH, ctx->h, s.D, Mmax, 64, P->qkv.tn)) != PAE_OK) return st;
  if (P->fuse_norm && (st = make_map_f32(ctx, &P->tmHg, ctx->h, s.D, Mmax, 64, P->gu.tn)) != PAE_OK) return st;
  return PAE_OK;
}

// Launch bracketing for PAE_OPT_PROFILE: events come from a pool sized before
// capture starts (ensure_events), so nothing is created during capture.
struct ProfScope {
  pae_ctx* ctx;
  cudaStream_t st;
  int kind, ev0 = -1;
  ProfScope(pae_ctx* c, int k, cudaStream_t s) : ctx(c), st(s), kind(k) {
    if ((ctx->profile_mask >> kind) & 1u) {
      if (ctx->ev_next + 2 <= (int)ctx->ev_pool.size() && ctx->rec_sink) {
        ev0 = ctx->ev_next;
        ctx->ev_next += 2;
        record(ctx->ev_pool[ev0]);
      }
    }
  }
  // Inside stream capture an event becomes a graph node only when recorded
  // as an external event.
  void record(cudaEvent_t e) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
      cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    else
      cudaEventRecord(e, st);
  }
  ~ProfScope() {
    if (ev0 >= 0) {
      record(ctx->ev_pool[ev0 + 1]);
      ctx->rec_sink->push_back(ProfRec{kind, ev0, ev0 + 1});
    }
  }
};

pae_status ensure_events(pae_ctx* ctx, int k_steps) {
  if (!ctx->profile_mask) return PAE_OK;
  const size_t need = (size_t)2 * ((size_t)k_steps * (7 * ctx->s.L + 1) + 3);
  while (ctx->ev_pool.size() < need) {
    cudaEvent_t e;
    CK(cudaEventCreate(&e));
    ctx->ev_pool.push_back(e);
  }
  return PAE_OK;
}

// PDL is used in the bf16 modes, and not while launches are bracketed by
// profiling events (an event between two kernels is not a kernel edge).
bool pdl_on(const pae_ctx* ctx) { return ctx->use_pdl && ctx->act_bf16 && ctx->profile_mask == 0; }

const float* tab(const pae_ctx* ctx, int k) { return ctx->tables + (size_t)k * ctx->s.table_rows; }

// `norm` (QKV and gate/up with P.fuse_norm): the step's scale / shift rows of
// that adaRMSNorm and how many sum-of-squares slots hold its statistics.
struct NormIn {
  const float* scale = nullptr;
  const float* shift = nullptr;
  int nslots = 0;
};

// Keep the first launch-helper error of the current enqueue_steps call.
void note_launch(pae_ctx* ctx, cudaError_t e) {
  if (e != cudaSuccess && ctx->enq_err == cudaSuccess) ctx->enq_err = e;
}

// The launch errors of the last enqueue_steps call: a helper's own refusal
// first, else the runtime's last error.
cudaError_t enqueue_error(pae_ctx* ctx) {
  const cudaError_t e = cudaGetLastError();
  return ctx->enq_err != cudaSuccess ? ctx->enq_err : e;
}

void run_gemm(pae_ctx* ctx, const Plan& P, int which, int layer, const EpiArgs& e, cudaStream_t st,
              const NormIn& norm = NormIn{}) {
  const Shape& s = ctx->s;
  const size_t es = ctx->esize;
  if (!ctx->act_bf16) {
    const float* X;
    const float* W;
    int N, K;
    switch (which) {
      case 0: X = (const float*)ctx->y; W = (const float*)((char*)ctx->w_qkv + (size_t)layer * s.qkv_rows * s.D * es); N = s.qkv_rows; K = s.D; break;
      case 1: X = (const float*)ctx->o; W = (const float*)((char*)ctx->w_o + (size_t)layer * s.D * s.attn_dim * es); N = s.D; K = s.attn_dim; break;
      case 2: X = (const float*)ctx->y; W = (const float*)((char*)ctx->w_gu + (size_t)layer * 2 * s.F * s.D * es); N = s.F; K = s.D; break;
      default: X = (const float*)ctx->u; W = (const float*)((char*)ctx->w_down + (size_t)layer * s.D * s.F * es); N = s.D; K = s.F; break;
    }
    launch_gemm_simple(s, X, W, N, K, e, st);
    return;
  }
  TcGemmArgs a{};
  a.e = e;
  a.err = DevErr{ctx->err_dev, ctx->wait_ns};
  const CUtensorMap *tw, *tx;
  const TcPlan* p;
  int na = 1;
  const bool w4 = ctx->w4 != 0;
  switch (which) {
    case 0: tw = w4 ? &ctx->tmQqkv : &ctx->tmWqkv; tx = &P.tmY; p = &P.qkv; a.N = s.qkv_rows; a.K = s.D;
            a.w_row0 = layer * s.qkv_rows; a.scales = (const bf16*)ctx->sc_qkv; break;
    case 1: tw = w4 ? &ctx->tmQo : &ctx->tmWo; tx = &P.tmO; p = &P.o; a.N = s.D; a.K = s.attn_dim;
            a.w_row0 = layer * s.D; a.scales = (const bf16*)ctx->sc_o; break;
    case 2: tw = w4 ? &ctx->tmQgu : &ctx->tmWgu; tx = &P.tmYg; p = &P.gu; a.N = s.F; a.K = s.D;
            a.w_row0 = layer * 2 * s.F; na = 2; a.scales = (const bf16*)ctx->sc_gu; break;
    default: tw = w4 ? &ctx->tmQdown : &ctx->tmWdown; tx = &P.tmU; p = &P.down; a.N = s.D; a.K = s.F;
             a.w_row0 = layer * s.D; a.scales = (const bf16*)ctx->sc_down; break;
  }
  if (!w4) a.scales = nullptr;
  if (norm.scale) {
    tx = which == 2 ? &P.tmHg : &P.tmH;
    a.ss_in = ctx->ss_buf;
    a.ss_ld = ctx->ss_ld;
    a.nslots = norm.nslots;
    a.nscale = norm.scale;
    a.nshift = norm.shift;
  }
  note_launch(ctx, launch_tc_gemm(s, tw, tx, na, *p, a, pdl_on(ctx), st));
}

// Enqueue Euler steps k_begin..k_end-1 for the plan's batch on `st`, with the
// state in ctx->x.
void enqueue_steps(pae_ctx* ctx, const Plan& P, int k_begin, int k_end, cudaStream_t st) {
  const Shape& s = ctx->s;
  const int M = P.M;
  ctx->enq_err = cudaSuccess;
  TransitionArgs ta{};
  ta.x = ctx->x;
  ta.x_src = ctx->x;
  ta.x_dst = ctx->x;
  ta.h = ctx->h;
  ta.y = ctx->y;
  ta.w_in = ctx->w_inT;
  ta.b_in = ctx->b_in;
  ta.w_out = ctx->w_out;
  ta.b_out = ctx->b_out;
  ta.dt = ctx->dt;
  ta.M = M;
  ta.ss_out = (P.fuse_norm || P.factored) ? ctx->ss_buf : nullptr;
  ta.y_factored = P.factored ? 1 : 0;
  ctx->ev_next = 0;
  const int slots_o = (s.D / 128) * P.o.splits, slots_down = (s.D / 128) * P.down.splits;
  // factored adaRMSNorm: one slot per (tile, rank, 32 rows)
  const int fslots_o = slots_o, fslots_down = slots_down;  // one slot per (tile, rank)
  for (int k = k_begin; k < k_end; ++k) {
    const float* tk = tab(ctx, k);
    ta.tab_out = (k == k_begin) ? nullptr : tab(ctx, k - 1);
    ta.k_out = k - 1;
    ta.tab_in = tk;
    {
      ProfScope ps(ctx, PAE_K_TRANSITION, st);
      note_launch(ctx, launch_transition(s, ctx->act_bf16, ta, pdl_on(ctx), st));
    }
    for (int l = 0; l < s.L; ++l) {
      EpiArgs e{};
      e.M = M;
      e.layer = l;
      e.epi = EPI_QKV;
      e.q = ctx->q;
      e.kc = ctx->kc;
      e.vc = ctx->vc;
      e.lens = ctx->lens_dev;
      e.rope_cs = ctx->rope_cs;
      if (P.factored) {
        e.f_bias = ctx->bias_qkv + ((size_t)k * s.L + l) * s.qkv_rows;
        e.f_ss = ctx->ss_buf;
        e.ss_ld = ctx->ss_ld;
        e.f_nslots = l == 0 ? 1 : fslots_down;
      }
      {
        ProfScope ps(ctx, PAE_K_QKV, st);
        NormIn nq;
        if (P.fuse_norm) nq = NormIn{tk + mod_offset(s, l, 0, 0), tk + mod_offset(s, l, 0, 1), l == 0 ? 1 : slots_down};
        run_gemm(ctx, P, 0, l, e, st, nq);
      }
      {
        ProfScope ps(ctx, PAE_K_ATTENTION, st);
        if (ctx->act_bf16) {
          AttnArgs aa{};
          aa.lens = ctx->lens_dev;
          aa.layer = l;
          aa.keys_per_split = P.attn.keys_per_split;
          aa.o = ctx->o;
          aa.part_o = static_cast<bf16*>(ctx->attn_part);
          aa.part_ml = reinterpret_cast<float2*>(static_cast<char*>(ctx->attn_part) +
                                                 (size_t)kAttnPartSlots * 128 * s.d * 2);
          aa.err = DevErr{ctx->err_dev, ctx->wait_ns};
          note_launch(ctx, launch_attn_tc(s, &ctx->tmQ, &ctx->tmK, &ctx->tmV, P.attn, aa, P.B, pdl_on(ctx), st));
        } else {
          launch_attention_simple(s, ctx->act_bf16, ctx->q, ctx->kc, ctx->vc, ctx->lens_dev, l, ctx->o, P.B, st);
        }
      }
      e = EpiArgs{};
      e.M = M;
      e.epi = EPI_RESID;
      e.h = ctx->h;
      e.gate = tk + mod_offset(s, l, 0, 2);
      if (P.fuse_norm || P.factored) {
        e.ss_out = ctx->ss_buf;
        e.ss_ld = ctx->ss_ld;
      }
      if (P.factored) {
        e.y_out = ctx->y;
        e.y_scale = tk + mod_offset(s, l, 1, 0);
      }
      {
        ProfScope ps(ctx, PAE_K_OPROJ, st);
        run_gemm(ctx, P, 1, l, e, st);
      }
      if (!P.fuse_norm && !P.factored) {
        ProfScope ps(ctx, PAE_K_NORM, st);
        note_launch(ctx, launch_norm(s, ctx->act_bf16, ctx->h, ctx->y, tk + mod_offset(s, l, 1, 0),
                                     tk + mod_offset(s, l, 1, 1), M, pdl_on(ctx), st));
      }
      e = EpiArgs{};
      e.M = M;
      e.epi = EPI_GEGLU;
      e.u = ctx->u;
      if (P.factored) {
        e.f_bias = ctx->bias_gu + ((size_t)k * s.L + l) * 2 * s.F;
        e.f_ss = ctx->ss_buf;
        e.ss_ld = ctx->ss_ld;
        e.f_nslots = fslots_o;
      }
      {
        ProfScope ps(ctx, PAE_K_GATEUP, st);
        NormIn ng;
        if (P.fuse_norm) ng = NormIn{tk + mod_offset(s, l, 1, 0), tk + mod_offset(s, l, 1, 1), slots_o};
        run_gemm(ctx, P, 2, l, e, st, ng);
      }
      e = EpiArgs{};
      e.M = M;
      e.epi = EPI_RESID;
      e.h = ctx->h;
      e.gate = tk + mod_offset(s, l, 1, 2);
      if (P.fuse_norm || (P.factored && l + 1 < s.L)) {
        e.ss_out = ctx->ss_buf;
        e.ss_ld = ctx->ss_ld;
      }
      if (P.factored && l + 1 < s.L) {
        e.y_out = ctx->y;
        e.y_scale = tk + mod_offset(s, l + 1, 0, 0);
      }
      {
        ProfScope ps(ctx, PAE_K_DOWN, st);
        run_gemm(ctx, P, 3, l, e, st);
      }
      if (l + 1 < s.L && !P.fuse_norm && !P.factored) {
        ProfScope ps(ctx, PAE_K_NORM, st);
        note_launch(ctx, launch_norm(s, ctx->act_bf16, ctx->h, ctx->y, tk + mod_offset(s, l + 1, 0, 0),
                                     tk + mod_offset(s, l + 1, 0, 1), M, pdl_on(ctx), st));
      }
    }
  }
  ta.tab_out = tab(ctx, k_end - 1);
  ta.k_out = k_end - 1;
  ta.tab_in = nullptr;
  {
    ProfScope ps(ctx, PAE_K_TRANSITION, st);
    note_launch(ctx, launch_transition(s, ctx->act_bf16, ta, pdl_on(ctx), st));
  }
}

pae_status get_plan(pae_ctx* ctx, int B, Plan** out) {
  auto it = ctx->plans.find(B);
  if (it == ctx->plans.end()) {
    Plan P;
    pae_status st = build_plan(ctx, B, &P);
    if (st != PAE_OK) return st;
    it = ctx->plans.emplace(B, P).first;
  }
  *out = &it->second;
  return PAE_OK;
}

void drop_graphs(pae_ctx* ctx) {
  for (auto& kv : ctx->plans) {
    if (kv.second.graph) cudaGraphExecDestroy(kv.second.graph);
    kv.second.graph = nullptr;
    kv.second.graph_K = 0;
  }
}

pae_status check_rows(pae_ctx* ctx, int batch) {
  for (int b = 0; b < batch; ++b)
    if (ctx->lens_host[b] < 0) return fail(ctx, PAE_ERR_STATE, "prefix row %d was never set", b);
  return PAE_OK;
}

bool use_persist(const pae_ctx* ctx, const Plan* P) { return ctx->use_persistent && P->persist; }
bool use_flow(const pae_ctx* ctx, const Plan* P) { return ctx->use_flow && P->flow && !use_persist(ctx, P); }

// Steps k_begin..k_end-1 (and the final Euler update) as one dataflow launch.
pae_status enqueue_flow(pae_ctx* ctx, Plan* P, int k_begin, int k_end, cudaStream_t st) {
  FlowArgs fa = P->fa;
  fa.k_begin = k_begin;
  fa.k_end = k_end;
  fa.err = DevErr{ctx->err_dev, ctx->wait_ns};
  const bool w4 = ctx->w4 != 0;
  const CUtensorMap maps[11] = {w4 ? ctx->tmQqkv : ctx->tmWqkv, w4 ? ctx->tmQo : ctx->tmWo,
                                w4 ? ctx->tmQg64 : ctx->tmWg64, w4 ? ctx->tmQdown : ctx->tmWdown,
                                ctx->tmYq64, ctx->tmO64, ctx->tmYg64, ctx->tmU64, ctx->tmQ, ctx->tmK, ctx->tmV};
  P->recs.clear();
  ctx->rec_sink = &P->recs;
  ctx->ev_next = 0;
  CK(cudaMemsetAsync(ctx->f_ctr, 0, sizeof(unsigned) * kFlowCtrWords, st));
  cudaError_t e;
  {
    ProfScope ps(ctx, PAE_K_DATAFLOW, st);
    e = launch_flow(ctx->s, maps, fa, st);
  }
  ctx->rec_sink = nullptr;
  if (e != cudaSuccess) return fail(ctx, PAE_ERR_CUDA, "dataflow launch: %s", cudaGetErrorString(e));
  return PAE_OK;
}

// Steps k_begin..k_end-1 (and the final Euler update) as one persistent launch.
pae_status enqueue_persistent(pae_ctx* ctx, Plan* P, int k_begin, int k_end, cudaStream_t st) {
  PersistArgs pa = P->pa;
  pa.k_begin = k_begin;
  pa.k_end = k_end;
  pa.err = DevErr{ctx->err_dev, ctx->wait_ns};
  const CUtensorMap maps[7] = {ctx->tmWqkv, ctx->tmWo, ctx->tmWgu1, ctx->tmWdown, ctx->tmQ, ctx->tmK, ctx->tmV};
  P->recs.clear();
  ctx->rec_sink = &P->recs;
  ctx->ev_next = 0;
  CK(cudaMemsetAsync(ctx->pw_ctr, 0, sizeof(unsigned) * kPersistCtrWords, st));
  cudaError_t e;
  {
    ProfScope ps(ctx, PAE_K_PERSISTENT, st);
    e = launch_persistent(ctx->s, maps, pa, st);
  }
  ctx->rec_sink = nullptr;
  if (e != cudaSuccess) return fail(ctx, PAE_ERR_CUDA, "persistent launch: %s", cudaGetErrorString(e));
  return PAE_OK;
}

pae_status run_loop(pae_ctx* ctx, Plan* P, cudaStream_t stream) {
  pae_status pst = ensure_events(ctx, ctx->K);
  if (pst != PAE_OK) return pst;
  ctx->last_plan = P;
  if (use_persist(ctx, P)) return enqueue_persistent(ctx, P, 0, ctx->K, stream);
  if (use_flow(ctx, P)) return enqueue_flow(ctx, P, 0, ctx->K, stream);
  if (!ctx->use_graph) {
    P->recs.clear();
    ctx->rec_sink = &P->recs;
    enqueue_steps(ctx, *P, 0, ctx->K, stream);
    ctx->rec_sink = nullptr;
    CK(enqueue_error(ctx));
    return PAE_OK;
  }
  if (!P->graph || P->graph_K != ctx->K) {
    if (P->graph) cudaGraphExecDestroy(P->graph);
    P->graph = nullptr;
    cudaGraph_t g = nullptr;
    P->recs.clear();
    ctx->rec_sink = &P->recs;
    CK(cudaStreamBeginCapture(ctx->cap_stream, cudaStreamCaptureModeThreadLocal));
    enqueue_steps(ctx, *P, 0, ctx->K, ctx->cap_stream);
    ctx->rec_sink = nullptr;
    cudaError_t e1 = enqueue_error(ctx);
    cudaError_t e2 = cudaStreamEndCapture(ctx->cap_stream, &g);
    if (e1 != cudaSuccess || e2 != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      return fail(ctx, PAE_ERR_CUDA, "graph capture failed: %s / %s", cudaGetErrorString(e1), cudaGetErrorString(e2));
    }
    size_t nn = 0;
    P->graph_kernels = 0;
    if (cudaGraphGetNodes(g, nullptr, &nn) == cudaSuccess && nn > 0) {
      std::vector<cudaGraphNode_t> nodes(nn);
      if (cudaGraphGetNodes(g, nodes.data(), &nn) == cudaSuccess)
        for (size_t i = 0; i < nn; ++i) {
          cudaGraphNodeType t;
          if (cudaGraphNodeGetType(nodes[i], &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++P->graph_kernels;
        }
    }
    cudaError_t e3 = cudaGraphInstantiate(&P->graph, g, 0);
    cudaGraphDestroy(g);
    if (e3 != cudaSuccess) {
      P->graph = nullptr;
      return fail(ctx, PAE_ERR_CUDA, "cudaGraphInstantiate: %s", cudaGetErrorString(e3));
    }
    P->graph_K = ctx->K;
  }
  CK(cudaGraphLaunch(P->graph, stream));
  return PAE_OK;
}

void free_all(pae_ctx* ctx) {
  if (!ctx) return;
  drop_graphs(ctx);
  for (cudaEvent_t e : ctx->ev_pool) cudaEventDestroy(e);
  ctx->ev_pool.clear();
  for (void* p : ctx->allocs) cudaFree(p);
  ctx->allocs.clear();
  if (ctx->err_host) cudaFreeHost(ctx->err_host);
  ctx->err_host = nullptr;
  if (ctx->cap_stream) cudaStreamDestroy(ctx->cap_stream);
  ctx->cap_stream = nullptr;
}

bool is_pos(int v) { return v > 0; }

Shape shape_from_config(const pae_config* cfg) {
  Shape s{};
  s.L = cfg->layers;
  s.D = cfg->width;
  s.Hq = cfg->n_q_heads;
  s.Hkv = cfg->n_kv_heads;
  s.d = cfg->head_dim;
  s.F = cfg->mlp_dim;
  s.A = cfg->action_dim;
  s.H = cfg->chunk;
  s.Bmax = cfg->max_batch;
  s.Pmax = cfg->max_prefix;
  s.Ptot = cfg->max_prefix + cfg->chunk;
  s.G = s.Hq / s.Hkv;
  s.qkv_rows = (s.Hq + 2 * s.Hkv) * s.d;
  s.attn_dim = s.Hq * s.d;
  s.group = cfg->group_size;
  s.eps = cfg->rms_eps;
  s.table_rows = (s.L * 2 * 3 + 2) * s.D;
  s.rope = cfg->rope_base > 0.f ? 1 : 0;
  s.Dp = cfg->prefix_width;
  return s;
}

pae_status validate_config(const pae_config* c) {
  if (!is_pos(c->layers) || !is_pos(c->width) || !is_pos(c->n_q_heads) || !is_pos(c->n_kv_heads) ||
      !is_pos(c->head_dim) || !is_pos(c->mlp_dim) || !is_pos(c->action_dim) || !is_pos(c->chunk) ||
      !is_pos(c->max_batch) || c->max_prefix < 0 || !(c->rms_eps > 0.f))
    return fail(nullptr, PAE_ERR_ARG, "config: sizes must be positive (max_prefix >= 0, rms_eps > 0)");
  if (c->dtype != PAE_FP32 && c->dtype != PAE_BF16 && c->dtype != PAE_W4A16)
    return fail(nullptr, PAE_ERR_ARG, "config: unknown dtype %d", c->dtype);
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: n_q_heads must be a multiple of n_kv_heads");
  if (c->n_q_heads / c->n_kv_heads > 16)
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: at most 16 query heads per KV head");
  if (c->width % 32 != 0 || c->width > 2048)
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: width must be a multiple of 32 and at most 2048");
  if (!(c->rope_base >= 0.f) || c->rope_base > 1e30f)
    return fail(nullptr, PAE_ERR_ARG, "config: rope_base must be 0 (off) or a finite positive base");
  if (c->rope_base > 0.f && c->head_dim % 2 != 0)
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: rotary embedding needs an even head_dim");
  if (c->prefix_width < 0) return fail(nullptr, PAE_ERR_ARG, "config: prefix_width must be >= 0");
  if (c->prefix_width > 0 && c->dtype != PAE_FP32 &&
      (c->prefix_width % 64 != 0 || (2 * c->n_kv_heads * c->head_dim) % 128 != 0))
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: bf16 prefix production needs prefix_width % 64 == 0 and "
                                              "2*n_kv_heads*head_dim % 128 == 0");
  if (c->dtype == PAE_W4A16 && c->group_size != 128)
    return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: W4A16 needs group_size 128");
  if (c->dtype != PAE_FP32) {
    const int qd = c->n_q_heads * c->head_dim;
    if (c->width % 128 || qd % 128 || c->mlp_dim % 128 || (c->n_kv_heads * c->head_dim) % 64)
      return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: bf16 kernels need width, n_q_heads*head_dim, mlp_dim "
                                                "multiples of 128");
    if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
      return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: bf16 attention needs head_dim 64, 128 or 256");
    if (c->chunk > 256 || (long long)c->max_batch * c->chunk > 4096)
      return fail(nullptr, PAE_ERR_UNSUPPORTED, "config: chunk <= 256 and max_batch*chunk <= 4096");
  }
  return PAE_OK;
}

// Launch plan of the prefix production GEMM: 128-token tiles (the height of
// the normalised-prefix tensor map's box) over `len` tokens, split-K so that
// output tiles x token tiles x splits fill the SMs.
TcPlan prefix_plan(const Shape& s, int len) {
  TcPlan p{};
  p.tn = 128;
  p.tok_tiles = (len + 127) / 128;
  const int nt = (2 * s.Hkv * s.d + 127) / 128, nkb = s.Dp / 64, base = nt * p.tok_tiles;
  p.splits = 1;
  for (int sp = 2; sp <= 8; sp *= 2)
    if (nkb % sp == 0 && base * sp <= 148) p.splits = sp;
  fit_ring(p, 1, nkb, false, false, 200u * 1024u);
  return p;
}

}  // namespace

extern "C" {

pae_status pae_create(const pae_config* cfg, const pae_weights* w, pae_ctx** out) {
  if (!out) return fail(nullptr, PAE_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg || !w) return fail(nullptr, PAE_ERR_ARG, "cfg or weights is NULL");
  pae_status st = validate_config(cfg);
  if (st != PAE_OK) return st;
  const void* req[] = {w->w_in, w->b_in, w->w_out, w->b_out, w->w_t1, w->b_t1, w->w_t2, w->b_t2,
                       w->w_mod, w->b_mod, w->w_modf, w->b_modf, w->w_qkv, w->w_o, w->w_gate, w->w_up, w->w_down};
  for (const void* p : req)
    if (!p) return fail(nullptr, PAE_ERR_ARG, "a required weight pointer is NULL");
  for (int l = 0; l < cfg->layers; ++l)
    if (!w->w_qkv[l] || !w->w_o[l] || !w->w_gate[l] || !w->w_up[l] || !w->w_down[l])
      return fail(nullptr, PAE_ERR_ARG, "layer %d weight pointer is NULL", l);
  if (cfg->dtype == PAE_W4A16) {
    if (!w->s_qkv || !w->s_o || !w->s_gate || !w->s_up || !w->s_down)
      return fail(nullptr, PAE_ERR_ARG, "W4A16 needs the s_* scale arrays");
    for (int l = 0; l < cfg->layers; ++l)
      if (!w->s_qkv[l] || !w->s_o[l] || !w->s_gate[l] || !w->s_up[l] || !w->s_down[l])
        return fail(nullptr, PAE_ERR_ARG, "layer %d scale pointer is NULL", l);
  }

  pae_ctx* ctx = new pae_ctx();
  ctx->cfg = *cfg;
  ctx->s = shape_from_config(cfg);
  Shape& s = ctx->s;
  ctx->act_bf16 = cfg->dtype != PAE_FP32;
  ctx->w4 = cfg->dtype == PAE_W4A16;
  ctx->esize = ctx->act_bf16 ? 2 : 4;
  const size_t es = ctx->esize;
  ctx->lens_host.assign(s.Bmax, -1);

  auto bail = [&](pae_status code) {
    g_create_error = ctx->last_error;
    free_all(ctx);
    delete ctx;
    return code;
  };
#define CKC(call)                                                                                   \
  do {                                                                                              \
    cudaError_t e_ = (call);                                                                        \
    if (e_ != cudaSuccess) {                                                                        \
      fail(ctx, PAE_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));                             \
      return bail(PAE_ERR_CUDA);                                                                    \
    }                                                                                               \
  } while (0)
#define ALLOC(ptr, bytes)                                                     \
  do {                                                                        \
    void* p_ = nullptr;                                                       \
    if ((st = dev_alloc(ctx, &p_, (bytes))) != PAE_OK) return bail(st);       \
    ptr = reinterpret_cast<decltype(ptr)>(p_);                                \
  } while (0)

  CKC(cudaGetDevice(&ctx->device));
  if (ctx->act_bf16) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    CKC(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (!fn || q != cudaDriverEntryPointSuccess) {
      fail(ctx, PAE_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
      return bail(PAE_ERR_CUDA);
    }
    ctx->encode = reinterpret_cast<EncodeTiledFn>(fn);
    CKC(tc_gemm_init());
  }
  CKC(cudaStreamCreateWithFlags(&ctx->cap_stream, cudaStreamNonBlocking));
  CKC(cudaHostAlloc(reinterpret_cast<void**>(&ctx->err_host), sizeof(int), cudaHostAllocMapped));
  *ctx->err_host = 0;
  CKC(cudaHostGetDevicePointer(reinterpret_cast<void**>(&ctx->err_dev), ctx->err_host, 0));

  const int L = s.L, D = s.D, A = s.A, F = s.F;
  // ---- weights
  ALLOC(ctx->w_inT, (size_t)D * A * es);
  ALLOC(ctx->b_in, (size_t)D * es);
  ALLOC(ctx->w_out, (size_t)A * D * es);
  ALLOC(ctx->b_out, (size_t)A * es);
  ALLOC(ctx->w_t1, (size_t)D * D * es);
  ALLOC(ctx->b_t1, (size_t)D * es);
  ALLOC(ctx->w_t2, (size_t)D * D * es);
  ALLOC(ctx->b_t2, (size_t)D * es);
  ALLOC(ctx->w_modall, (size_t)s.table_rows * D * es);
  ALLOC(ctx->b_modall, (size_t)s.table_rows * es);
  if (!ctx->w4) {
    ALLOC(ctx->w_qkv, (size_t)L * s.qkv_rows * D * es);
    ALLOC(ctx->w_o, (size_t)L * D * s.attn_dim * es);
    ALLOC(ctx->w_gu, (size_t)L * 2 * F * D * es);
    ALLOC(ctx->w_down, (size_t)L * D * F * es);
  } else {
    ALLOC(ctx->q_qkv, (size_t)L * s.qkv_rows * D / 2);
    ALLOC(ctx->q_o, (size_t)L * D * s.attn_dim / 2);
    ALLOC(ctx->q_gu, (size_t)L * 2 * F * D / 2);
    ALLOC(ctx->q_down, (size_t)L * D * F / 2);
    ALLOC(ctx->sc_qkv, (size_t)L * s.qkv_rows * (D / 128) * 2);
    ALLOC(ctx->sc_o, (size_t)L * D * (s.attn_dim / 128) * 2);
    ALLOC(ctx->sc_gu, (size_t)L * 2 * F * (D / 128) * 2);
    ALLOC(ctx->sc_down, (size_t)L * D * (F / 128) * 2);
  }
  cudaStream_t cs = ctx->cap_stream;
  if (ctx->act_bf16)
    k_transpose<uint16_t><<<64, 256, 0, cs>>>((const uint16_t*)w->w_in, (uint16_t*)ctx->w_inT, D, A);
  else
    k_transpose<float><<<64, 256, 0, cs>>>((const float*)w->w_in, (float*)ctx->w_inT, D, A);
  CKC(cudaGetLastError());
  CKC(cudaMemcpyAsync(ctx->b_in, w->b_in, (size_t)D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->w_out, w->w_out, (size_t)A * D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->b_out, w->b_out, (size_t)A * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->w_t1, w->w_t1, (size_t)D * D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->b_t1, w->b_t1, (size_t)D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->w_t2, w->w_t2, (size_t)D * D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->b_t2, w->b_t2, (size_t)D * es, cudaMemcpyDeviceToDevice, cs));
  const size_t mod_rows = (size_t)L * 2 * 3 * D;
  CKC(cudaMemcpyAsync(ctx->w_modall, w->w_mod, mod_rows * D * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync((char*)ctx->w_modall + mod_rows * D * es, w->w_modf, (size_t)2 * D * D * es,
                      cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync(ctx->b_modall, w->b_mod, mod_rows * es, cudaMemcpyDeviceToDevice, cs));
  CKC(cudaMemcpyAsync((char*)ctx->b_modall + mod_rows * es, w->b_modf, (size_t)2 * D * es,
                      cudaMemcpyDeviceToDevice, cs));
  for (int l = 0; l < L && ctx->w4; ++l) {
    const int rot_rows = s.rope ? (s.Hq + s.Hkv) * s.d : 0;
    auto rep = [&](const void* src, void* dst, int rows, int K, int mode, int rot = 0) {
      k_repack_int4<<<256, 256, 0, cs>>>((const uint8_t*)src, (uint8_t*)dst, rows, K / 2, mode, rot, s.d);
    };
    rep(w->w_qkv[l], (char*)ctx->q_qkv + (size_t)l * s.qkv_rows * D / 2, s.qkv_rows, D, 0, rot_rows);
    rep(w->w_o[l], (char*)ctx->q_o + (size_t)l * D * s.attn_dim / 2, D, s.attn_dim, 0);
    rep(w->w_down[l], (char*)ctx->q_down + (size_t)l * D * F / 2, D, F, 0);
    rep(w->w_gate[l], (char*)ctx->q_gu + (size_t)l * 2 * F * D / 2, F, D, 1);
    rep(w->w_up[l], (char*)ctx->q_gu + (size_t)l * 2 * F * D / 2, F, D, 2);
    CKC(cudaGetLastError());
    const size_t g1 = D / 128, g2 = s.attn_dim / 128, g3 = F / 128;
    if (s.rope)
      k_permute_rows<<<64, 256, 0, cs>>>((const uint16_t*)w->s_qkv[l],
                                         (uint16_t*)((char*)ctx->sc_qkv + (size_t)l * s.qkv_rows * g1 * 2), s.qkv_rows,
                                         (int)g1, rot_rows, s.d);
    else
      CKC(cudaMemcpyAsync((char*)ctx->sc_qkv + (size_t)l * s.qkv_rows * g1 * 2, w->s_qkv[l],
                          (size_t)s.qkv_rows * g1 * 2, cudaMemcpyDeviceToDevice, cs));
    CKC(cudaGetLastError());
    CKC(cudaMemcpyAsync((char*)ctx->sc_o + (size_t)l * D * g2 * 2, w->s_o[l], (size_t)D * g2 * 2,
                        cudaMemcpyDeviceToDevice, cs));
    CKC(cudaMemcpyAsync((char*)ctx->sc_down + (size_t)l * D * g3 * 2, w->s_down[l], (size_t)D * g3 * 2,
                        cudaMemcpyDeviceToDevice, cs));
    char* gu = (char*)ctx->sc_gu + (size_t)l * 2 * F * g1 * 2;
    const size_t tile = (size_t)128 * g1 * 2;
    CKC(cudaMemcpy2DAsync(gu, 2 * tile, w->s_gate[l], tile, tile, F / 128, cudaMemcpyDeviceToDevice, cs));
    CKC(cudaMemcpy2DAsync(gu + tile, 2 * tile, w->s_up[l], tile, tile, F / 128, cudaMemcpyDeviceToDevice, cs));
  }
  for (int l = 0; l < L && !ctx->w4; ++l) {
    if (s.rope)
      k_permute_rows<<<256, 256, 0, cs>>>((const uint16_t*)w->w_qkv[l],
                                          (uint16_t*)((char*)ctx->w_qkv + (size_t)l * s.qkv_rows * D * es), s.qkv_rows,
                                          (int)(D * es / 2), (s.Hq + s.Hkv) * s.d, s.d);
    else
      CKC(cudaMemcpyAsync((char*)ctx->w_qkv + (size_t)l * s.qkv_rows * D * es, w->w_qkv[l],
                          (size_t)s.qkv_rows * D * es, cudaMemcpyDeviceToDevice, cs));
    CKC(cudaGetLastError());
    CKC(cudaMemcpyAsync((char*)ctx->w_o + (size_t)l * D * s.attn_dim * es, w->w_o[l], (size_t)D * s.attn_dim * es,
                        cudaMemcpyDeviceToDevice, cs));
    CKC(cudaMemcpyAsync((char*)ctx->w_down + (size_t)l * D * F * es, w->w_down[l], (size_t)D * F * es,
                        cudaMemcpyDeviceToDevice, cs));
    // gate/up interleaved in 128-row tiles: [gate 128 rows | up 128 rows] per tile
    char* gu = (char*)ctx->w_gu + (size_t)l * 2 * F * D * es;
    const size_t tile_bytes = (size_t)128 * D * es;
    const int full_tiles = F / 128;
    if (full_tiles > 0) {
      CKC(cudaMemcpy2DAsync(gu, 2 * tile_bytes, w->w_gate[l], tile_bytes, tile_bytes, full_tiles,
                            cudaMemcpyDeviceToDevice, cs));
      CKC(cudaMemcpy2DAsync(gu + tile_bytes, 2 * tile_bytes, w->w_up[l], tile_bytes, tile_bytes, full_tiles,
                            cudaMemcpyDeviceToDevice, cs));
    }
    const int rem = F - full_tiles * 128;  // fp32 mode only (bf16 needs F % 128 == 0)
    if (rem > 0) {
      const size_t rb = (size_t)rem * D * es;
      CKC(cudaMemcpyAsync(gu + full_tiles * 2 * tile_bytes, (const char*)w->w_gate[l] + full_tiles * tile_bytes, rb,
                          cudaMemcpyDeviceToDevice, cs));
      CKC(cudaMemcpyAsync(gu + full_tiles * 2 * tile_bytes + tile_bytes,
                          (const char*)w->w_up[l] + full_tiles * tile_bytes, rb, cudaMemcpyDeviceToDevice, cs));
    }
  }
  // ---- tables, prefix slots, activations
  ALLOC(ctx->t_dev, sizeof(double) * (kMaxSteps + 1));
  ALLOC(ctx->emb, sizeof(float) * kMaxSteps * D);
  ALLOC(ctx->zbuf, sizeof(float) * kMaxSteps * D);
  ALLOC(ctx->cbuf, sizeof(float) * kMaxSteps * D);
  ALLOC(ctx->tables, sizeof(float) * kMaxSteps * (size_t)s.table_rows);
  ALLOC(ctx->dt, sizeof(float) * kMaxSteps);
  const size_t slot_elems = (size_t)L * s.Bmax * s.Hkv * s.Ptot * s.d;
  ALLOC(ctx->kc, slot_elems * es);
  ALLOC(ctx->vc, slot_elems * es);
  CKC(cudaMemsetAsync(ctx->kc, 0, slot_elems * es, cs));
  CKC(cudaMemsetAsync(ctx->vc, 0, slot_elems * es, cs));
  if (s.rope) {
    // (cos, sin) per position and channel pair, angles in float64 from the
    // integer positions, each rounded once to fp32
    const int half = s.d / 2;
    std::vector<float2> cs_host((size_t)s.Ptot * half);
    for (int pos = 0; pos < s.Ptot; ++pos)
      for (int i = 0; i < half; ++i) {
        const double a = (double)pos * std::pow((double)cfg->rope_base, -2.0 * i / (double)s.d);
        cs_host[(size_t)pos * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    ALLOC(ctx->rope_cs, sizeof(float2) * cs_host.size());
    CKC(cudaMemcpyAsync(ctx->rope_cs, cs_host.data(), sizeof(float2) * cs_host.size(), cudaMemcpyHostToDevice, cs));
    CKC(cudaStreamSynchronize(cs));  // cs_host goes out of scope
  }
  if (s.Dp > 0) {
    const int kvr = 2 * s.Hkv * s.d;
    ALLOC(ctx->w_pkv, (size_t)L * kvr * s.Dp * es);
    ALLOC(ctx->ypre, (size_t)std::max(s.Pmax, 1) * s.Dp * es);
    for (int l = 0; l < L; ++l) {
      if (!w->w_prefix_kv || !w->w_prefix_kv[l]) {
        fail(ctx, PAE_ERR_ARG, "prefix_width > 0 needs w_prefix_kv for every layer");
        return bail(PAE_ERR_ARG);
      }
      k_permute_rows<<<256, 256, 0, cs>>>((const uint16_t*)w->w_prefix_kv[l],
                                          (uint16_t*)((char*)ctx->w_pkv + (size_t)l * kvr * s.Dp * es), kvr,
                                          (int)(s.Dp * es / 2), s.rope ? s.Hkv * s.d : 0, s.d);
      CKC(cudaGetLastError());
    }
    if (ctx->act_bf16) {
      if ((st = make_map(ctx, &ctx->tmWpkv, ctx->w_pkv, s.Dp, (uint64_t)L * kvr, 64, 128)) != PAE_OK) return bail(st);
      if ((st = make_map(ctx, &ctx->tmYpre, ctx->ypre, s.Dp, (uint64_t)std::max(s.Pmax, 1), 64, 128)) != PAE_OK)
        return bail(st);
    }
  }
  ALLOC(ctx->lens_dev, sizeof(int) * s.Bmax);
  CKC(cudaMemsetAsync(ctx->lens_dev, 0, sizeof(int) * s.Bmax, cs));
  const size_t Mmax = (size_t)s.Bmax * s.H;
  const size_t Mpad = ((Mmax + 255) / 256 + 1) * 256;  // token tiles may pad past Mmax
  ALLOC(ctx->x, sizeof(float) * Mmax * A);
  ALLOC(ctx->h, sizeof(float) * Mmax * D);
  ALLOC(ctx->y, Mpad * D * es);
  ALLOC(ctx->q, Mmax * s.attn_dim * es);
  ALLOC(ctx->o, Mpad * s.attn_dim * es);
  ALLOC(ctx->u, Mpad * F * es);
  CKC(cudaMemsetAsync(ctx->y, 0, Mpad * D * es, cs));
  CKC(cudaMemsetAsync(ctx->o, 0, Mpad * s.attn_dim * es, cs));
  CKC(cudaMemsetAsync(ctx->u, 0, Mpad * F * es, cs));
  ctx->ss_ld = (int)Mpad;
  ALLOC(ctx->ss_buf, sizeof(float) * kSsSlots * Mpad);
  CKC(cudaMemsetAsync(ctx->ss_buf, 0, sizeof(float) * kSsSlots * Mpad, cs));
  if (ctx->act_bf16) {
    const size_t part_bytes = (size_t)kAttnPartSlots * 128 * (s.d * 2 + 8);
    ALLOC(ctx->attn_part, part_bytes);
    CKC(cudaMemsetAsync(ctx->attn_part, 0, part_bytes, cs));
  }
  if (ctx->act_bf16 && !ctx->w4) {
    if ((st = make_map(ctx, &ctx->tmWqkv, ctx->w_qkv, D, (uint64_t)L * s.qkv_rows, 64, 128)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmWo, ctx->w_o, s.attn_dim, (uint64_t)L * D, 64, 128)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmWgu, ctx->w_gu, D, (uint64_t)L * 2 * F, 64, 256)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmWdown, ctx->w_down, F, (uint64_t)L * D, 64, 128)) != PAE_OK) return bail(st);
  }
  if (ctx->w4) {
    if ((st = make_map_u8(ctx, &ctx->tmQqkv, ctx->q_qkv, D / 2, (uint64_t)L * s.qkv_rows, 32, 128)) != PAE_OK)
      return bail(st);
    if ((st = make_map_u8(ctx, &ctx->tmQo, ctx->q_o, s.attn_dim / 2, (uint64_t)L * D, 32, 128)) != PAE_OK)
      return bail(st);
    if ((st = make_map_u8(ctx, &ctx->tmQgu, ctx->q_gu, D / 2, (uint64_t)L * 2 * F, 32, 256)) != PAE_OK)
      return bail(st);
    if ((st = make_map_u8(ctx, &ctx->tmQdown, ctx->q_down, F / 2, (uint64_t)L * D, 32, 128)) != PAE_OK)
      return bail(st);
    if ((st = make_map_u8(ctx, &ctx->tmQg64, ctx->q_gu, D / 2, (uint64_t)L * 2 * F, 32, 64)) != PAE_OK)
      return bail(st);
  }
  if (ctx->act_bf16 && !ctx->w4) {
    // persistent kernel: 128-row gate/up boxes, workspace, one CTA per SM
    if ((st = make_map(ctx, &ctx->tmWgu1, ctx->w_gu, D, (uint64_t)L * 2 * F, 64, 128)) != PAE_OK) return bail(st);
    CKC(persist_init());
    int nsm = 0;
    CKC(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, ctx->device));
    int coop = 0;
    CKC(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, ctx->device));
    ctx->ncta = coop ? nsm : 0;
    const size_t part = (size_t)nsm * std::max<size_t>(128 * 64, (size_t)128 * s.d + 256);
    ALLOC(ctx->pw_part, sizeof(float) * part);
    ALLOC(ctx->pw_ss, sizeof(float) * kPersistGroups * 64);
    ALLOC(ctx->pw_ctr, sizeof(unsigned) * kPersistCtrWords);
  }
  if (ctx->act_bf16) {
    // dataflow loop: buffers, 64-row operand maps, occupancy of each cluster size
    ctx->flow_capable = true;
    CKC(flow_init());
    for (int C : {2, 4, 8, 16}) ctx->flow_max_cl[C] = flow_max_clusters(C);
    ALLOC(ctx->yg, Mpad * D * es);
    CKC(cudaMemsetAsync(ctx->yg, 0, Mpad * D * es, cs));
    ALLOC(ctx->f_ssq, sizeof(float) * (size_t)(D / 128) * 16 * 64);
    ALLOC(ctx->f_ssg, sizeof(float) * (size_t)(D / 128) * 16 * 64);
    ALLOC(ctx->f_sst, sizeof(float) * 64);
    ALLOC(ctx->bias_qkv, sizeof(float) * (size_t)kMaxSteps * L * s.qkv_rows);
    ALLOC(ctx->bias_gu, sizeof(float) * (size_t)kMaxSteps * L * 2 * F);
    ALLOC(ctx->f_ctr, sizeof(unsigned) * kFlowCtrWords);
    if (!ctx->w4 && (st = make_map(ctx, &ctx->tmWg64, ctx->w_gu, D, (uint64_t)L * 2 * F, 64, 64)) != PAE_OK)
      return bail(st);
    if ((st = make_map(ctx, &ctx->tmYq64, ctx->y, D, Mmax, 64, 64)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmYg64, ctx->yg, D, Mmax, 64, 64)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmO64, ctx->o, s.attn_dim, Mmax, 64, 64)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmU64, ctx->u, F, Mmax, 64, 64)) != PAE_OK) return bail(st);
  }
  if (ctx->act_bf16) {
    CKC(attn_tc_init());
    const uint64_t kv_rows = (uint64_t)L * s.Bmax * s.Hkv * s.Ptot;
    if ((st = make_map(ctx, &ctx->tmQ, ctx->q, s.d, (uint64_t)s.Bmax * s.Hq * s.H, 64, 128)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmK, ctx->kc, s.d, kv_rows, 64, 64)) != PAE_OK) return bail(st);
    if ((st = make_map(ctx, &ctx->tmV, ctx->vc, s.d, kv_rows, 64, 64)) != PAE_OK) return bail(st);
  }
  CKC(cudaStreamSynchronize(cs));
  CKC(cudaGetLastError());
  *out = ctx;
  return PAE_OK;
#undef CKC
#undef ALLOC
}

pae_status pae_set_prefix(pae_ctx* ctx, int row, const void* const* k_per_layer, const void* const* v_per_layer,
                          int len, pae_stream stream) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  pae_status st = check_err_word(ctx);
  if (st != PAE_OK) return st;
  const Shape& s = ctx->s;
  if (row < 0 || row >= s.Bmax) return fail(ctx, PAE_ERR_ARG, "row %d out of range [0, %d)", row, s.Bmax);
  if (len < 0 || len > s.Pmax) return fail(ctx, PAE_ERR_ARG, "len %d out of range [0, %d]", len, s.Pmax);
  if (len > 0) {
    if (!k_per_layer || !v_per_layer) return fail(ctx, PAE_ERR_ARG, "k/v pointer arrays are NULL");
    for (int l = 0; l < s.L; ++l)
      if (!k_per_layer[l] || !v_per_layer[l]) return fail(ctx, PAE_ERR_ARG, "layer %d k/v pointer is NULL", l);
  }
  cudaStream_t stm = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = ctx->esize;
  const size_t rowb = (size_t)s.d * es;
  for (int l = 0; l < s.L && len > 0; ++l) {
    for (int g = 0; g < s.Hkv; ++g) {
      const size_t slot = (((size_t)l * s.Bmax + row) * s.Hkv + g) * s.Ptot * s.d * es;
      const char* ks = static_cast<const char*>(k_per_layer[l]) + g * rowb;
      const char* vs = static_cast<const char*>(v_per_layer[l]) + g * rowb;
      CK(cudaMemcpy2DAsync((char*)ctx->kc + slot, rowb, ks, s.Hkv * rowb, rowb, len, cudaMemcpyDeviceToDevice, stm));
      CK(cudaMemcpy2DAsync((char*)ctx->vc + slot, rowb, vs, s.Hkv * rowb, rowb, len, cudaMemcpyDeviceToDevice, stm));
    }
  }
  k_set_len<<<1, 1, 0, stm>>>(ctx->lens_dev, row, len);
  CK(cudaGetLastError());
  ctx->lens_host[row] = len;
  return PAE_OK;
}

pae_status pae_set_prefix_hidden(pae_ctx* ctx, int row, const void* const* h_per_layer, int len,
                                 pae_stream stream) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  pae_status st = check_err_word(ctx);
  if (st != PAE_OK) return st;
  const Shape& s = ctx->s;
  if (s.Dp <= 0) return fail(ctx, PAE_ERR_STATE, "the context was created with prefix_width = 0");
  if (row < 0 || row >= s.Bmax) return fail(ctx, PAE_ERR_ARG, "row %d out of range [0, %d)", row, s.Bmax);
  if (len < 0 || len > s.Pmax) return fail(ctx, PAE_ERR_ARG, "len %d out of range [0, %d]", len, s.Pmax);
  if (len > 0) {
    if (!h_per_layer) return fail(ctx, PAE_ERR_ARG, "h_per_layer is NULL");
    for (int l = 0; l < s.L; ++l)
      if (!h_per_layer[l]) return fail(ctx, PAE_ERR_ARG, "layer %d hidden-state pointer is NULL", l);
  }
  cudaStream_t stm = reinterpret_cast<cudaStream_t>(stream);
  const int kvr = 2 * s.Hkv * s.d;
  const TcPlan plan = ctx->act_bf16 && len > 0 ? prefix_plan(s, len) : TcPlan{};
  for (int l = 0; l < s.L && len > 0; ++l) {
    CK(launch_prefix_norm(ctx->act_bf16, h_per_layer[l], ctx->ypre, len, s.Dp, s.eps, stm));
    EpiArgs e{};
    e.epi = EPI_PREFIX;
    e.M = len;
    e.kc = ctx->kc;
    e.vc = ctx->vc;
    e.layer = l;
    e.prefix_row = row;
    e.rope_cs = ctx->rope_cs;
    if (!ctx->act_bf16) {
      launch_gemm_simple(s, static_cast<const float*>(ctx->ypre),
                         static_cast<const float*>(ctx->w_pkv) + (size_t)l * kvr * s.Dp, kvr, s.Dp, e, stm);
    } else {
      TcGemmArgs a{};
      a.e = e;
      a.N = kvr;
      a.K = s.Dp;
      a.w_row0 = l * kvr;
      a.err = DevErr{ctx->err_dev, ctx->wait_ns};
      CK(launch_tc_gemm(s, &ctx->tmWpkv, &ctx->tmYpre, 1, plan, a, false, stm));
    }
    CK(cudaGetLastError());
  }
  k_set_len<<<1, 1, 0, stm>>>(ctx->lens_dev, row, len);
  CK(cudaGetLastError());
  ctx->lens_host[row] = len;
  return PAE_OK;
}

pae_status pae_precompute_tables(pae_ctx* ctx, const double* t, int K, pae_stream stream) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  pae_status st = check_err_word(ctx);
  if (st != PAE_OK) return st;
  if (!t) return fail(ctx, PAE_ERR_ARG, "t is NULL");
  if (K < 1 || K > kMaxSteps) return fail(ctx, PAE_ERR_ARG, "K = %d out of range [1, %d]", K, kMaxSteps);
  const double dir = t[1] - t[0];
  for (int k = 0; k < K; ++k) {
    const double dk = t[k + 1] - t[k];
    if (!(dk * dir > 0.0)) return fail(ctx, PAE_ERR_ARG, "t must be strictly monotone (at index %d)", k);
  }
  cudaStream_t stm = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(ctx->t_dev, t, sizeof(double) * (K + 1), cudaMemcpyHostToDevice, stm));
  launch_time_mlp(ctx->s, ctx->act_bf16, ctx->t_dev, K, ctx->w_t1, ctx->b_t1, ctx->w_t2, ctx->b_t2, ctx->emb,
                  ctx->zbuf, ctx->cbuf, ctx->dt, stm);
  launch_mod_tables(ctx->s, ctx->act_bf16, ctx->cbuf, K, ctx->w_modall, ctx->b_modall, ctx->tables, stm);
  if (ctx->flow_capable) {
    // the adaRMSNorm shifts projected through W_qkv and W_gate/up, per step and layer
    if (ctx->w4) {
      launch_shift_bias_w4(ctx->s, ctx->q_qkv, ctx->sc_qkv, ctx->s.qkv_rows, 0, ctx->tables, K, ctx->bias_qkv, stm);
      launch_shift_bias_w4(ctx->s, ctx->q_gu, ctx->sc_gu, 2 * ctx->s.F, 1, ctx->tables, K, ctx->bias_gu, stm);
    } else {
      launch_shift_bias(ctx->s, ctx->w_qkv, ctx->s.qkv_rows, 0, ctx->tables, K, ctx->bias_qkv, stm);
      launch_shift_bias(ctx->s, ctx->w_gu, 2 * ctx->s.F, 1, ctx->tables, K, ctx->bias_gu, stm);
    }
  }
  CK(cudaGetLastError());
  if (K != ctx->K) drop_graphs(ctx);
  ctx->K = K;
  ctx->tables_ready = true;
  return PAE_OK;
}

static pae_status denoise_common(pae_ctx* ctx, const float* noise, float* out, int batch, pae_stream stream,
                                 cudaMemcpyKind in_kind, cudaMemcpyKind out_kind) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  pae_status st = check_err_word(ctx);
  if (st != PAE_OK) return st;
  if (batch < 0 || batch > ctx->s.Bmax) return fail(ctx, PAE_ERR_ARG, "batch %d out of range [0, %d]", batch, ctx->s.Bmax);
  if (batch == 0) return PAE_OK;
  if (!noise || !out) return fail(ctx, PAE_ERR_ARG, "noise or out is NULL");
  if (!ctx->tables_ready) return fail(ctx, PAE_ERR_STATE, "pae_precompute_tables has not been called");
  if ((st = check_rows(ctx, batch)) != PAE_OK) return st;
  Plan* P = nullptr;
  if ((st = get_plan(ctx, batch, &P)) != PAE_OK) return st;
  cudaStream_t stm = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(float) * (size_t)batch * ctx->s.H * ctx->s.A;
  CK(cudaMemcpyAsync(ctx->x, noise, bytes, in_kind, stm));
  if ((st = run_loop(ctx, P, stm)) != PAE_OK) return st;
  CK(cudaMemcpyAsync(out, ctx->x, bytes, out_kind, stm));
  return PAE_OK;
}

pae_status pae_denoise(pae_ctx* ctx, const float* noise, float* out, int batch, pae_stream stream) {
  return denoise_common(ctx, noise, out, batch, stream, cudaMemcpyDeviceToDevice, cudaMemcpyDeviceToDevice);
}

pae_status pae_denoise_host(pae_ctx* ctx, const float* noise_host, float* out_host, int batch, pae_stream stream) {
  return denoise_common(ctx, noise_host, out_host, batch, stream, cudaMemcpyHostToDevice, cudaMemcpyDeviceToHost);
}

pae_status pae_denoise_steps(pae_ctx* ctx, const float* x_in, float* x_out, int batch, int k_begin, int k_end,
                             pae_stream stream) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  pae_status st = check_err_word(ctx);
  if (st != PAE_OK) return st;
  if (batch < 0 || batch > ctx->s.Bmax) return fail(ctx, PAE_ERR_ARG, "batch %d out of range [0, %d]", batch, ctx->s.Bmax);
  if (!ctx->tables_ready) return fail(ctx, PAE_ERR_STATE, "pae_precompute_tables has not been called");
  if (k_begin < 0 || k_end > ctx->K || k_begin >= k_end)
    return fail(ctx, PAE_ERR_ARG, "step range [%d, %d) invalid for K = %d", k_begin, k_end, ctx->K);
  if (batch == 0) return PAE_OK;
  if (!x_in || !x_out) return fail(ctx, PAE_ERR_ARG, "x_in or x_out is NULL");
  if ((st = check_rows(ctx, batch)) != PAE_OK) return st;
  Plan* P = nullptr;
  if ((st = get_plan(ctx, batch, &P)) != PAE_OK) return st;
  cudaStream_t stm = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(float) * (size_t)batch * ctx->s.H * ctx->s.A;
  if ((st = ensure_events(ctx, k_end - k_begin)) != PAE_OK) return st;
  CK(cudaMemcpyAsync(ctx->x, x_in, bytes, cudaMemcpyDeviceToDevice, stm));
  ctx->last_plan = P;
  if (use_persist(ctx, P)) {
    if ((st = enqueue_persistent(ctx, P, k_begin, k_end, stm)) != PAE_OK) return st;
  } else if (use_flow(ctx, P)) {
    if ((st = enqueue_flow(ctx, P, k_begin, k_end, stm)) != PAE_OK) return st;
  } else {
    P->recs.clear();
    ctx->rec_sink = &P->recs;
    enqueue_steps(ctx, *P, k_begin, k_end, stm);
    ctx->rec_sink = nullptr;
    CK(enqueue_error(ctx));
  }
  CK(cudaGetLastError());
  CK(cudaMemcpyAsync(x_out, ctx->x, bytes, cudaMemcpyDeviceToDevice, stm));
  return PAE_OK;
}

pae_status pae_set_option(pae_ctx* ctx, int option, long long value) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  switch (option) {
    case PAE_OPT_USE_GRAPH: ctx->use_graph = value != 0; return PAE_OK;
    case PAE_OPT_WAIT_LIMIT_US:
      if (value <= 0) return fail(ctx, PAE_ERR_ARG, "wait limit must be positive");
      ctx->wait_ns = value * 1000LL;
      drop_graphs(ctx);  // captured launches hold the old limit
      return PAE_OK;
    case PAE_OPT_MAX_SPLITK:
      if (value < 1 || value > 16) return fail(ctx, PAE_ERR_ARG, "max split-K must be in [1, 16]");
      if ((int)value != ctx->max_splitk) {
        drop_graphs(ctx);
        ctx->plans.clear();
        ctx->last_plan = nullptr;
      }
      ctx->max_splitk = (int)value;
      return PAE_OK;
    case PAE_OPT_PDL:
      if ((value != 0) != ctx->use_pdl) drop_graphs(ctx);
      ctx->use_pdl = value != 0;
      return PAE_OK;
    case PAE_OPT_PERSISTENT: ctx->use_persistent = value != 0; return PAE_OK;
    case PAE_OPT_DATAFLOW: ctx->use_flow = value != 0; return PAE_OK;
    case PAE_OPT_DATAFLOW_CLUSTER:
      if (value != 0 && value != 2 && value != 4 && value != 8 && value != 16)
        return fail(ctx, PAE_ERR_ARG, "dataflow cluster size must be 0 (automatic), 2, 4, 8 or 16");
      if ((int)value != ctx->flow_cluster) {
        drop_graphs(ctx);
        ctx->plans.clear();
        ctx->last_plan = nullptr;
      }
      ctx->flow_cluster = (int)value;
      return PAE_OK;
    case PAE_OPT_FUSED_NORM:
      if ((value != 0) != ctx->use_fused_norm) {
        drop_graphs(ctx);
        ctx->plans.clear();
        ctx->last_plan = nullptr;
      }
      ctx->use_fused_norm = value != 0;
      return PAE_OK;
    case PAE_OPT_FACTORED_NORM:
      if ((value != 0) != ctx->use_factored) {
        drop_graphs(ctx);
        ctx->plans.clear();
        ctx->last_plan = nullptr;
      }
      ctx->use_factored = value != 0;
      return PAE_OK;
    case PAE_OPT_PROFILE:
      if (value < 0 || value >= (1LL << PAE_K_COUNT)) return fail(ctx, PAE_ERR_ARG, "bad profile mask");
      if ((unsigned)value != ctx->profile_mask) drop_graphs(ctx);
      ctx->profile_mask = (unsigned)value;
      return PAE_OK;
    default: return fail(ctx, PAE_ERR_ARG, "unknown option %d", option);
  }
}

pae_status pae_profile_read(pae_ctx* ctx, int kernel_class, double* total_ms, int* launches) {
  if (!ctx || !total_ms || !launches) return fail(ctx, PAE_ERR_ARG, "null argument");
  if (kernel_class < 0 || kernel_class >= PAE_K_COUNT) return fail(ctx, PAE_ERR_ARG, "bad kernel class");
  *total_ms = 0.0;
  *launches = 0;
  if (!ctx->last_plan) return PAE_OK;
  for (const ProfRec& r : ctx->last_plan->recs) {
    if (r.kind != kernel_class) continue;
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, ctx->ev_pool[r.ev0], ctx->ev_pool[r.ev1]));
    *total_ms += ms;
    ++*launches;
  }
  return PAE_OK;
}

pae_status pae_query(pae_ctx* ctx, int what, int batch, long long* value) {
  if (!ctx || !value) return fail(ctx, PAE_ERR_ARG, "null argument");
  if (batch < 1 || batch > ctx->s.Bmax) return fail(ctx, PAE_ERR_ARG, "batch %d out of range", batch);
  Plan* P = nullptr;
  pae_status st = get_plan(ctx, batch, &P);
  if (st != PAE_OK) return st;
  switch (what) {
    case PAE_Q_GRAPH_KERNELS: *value = P->graph ? P->graph_kernels : 0; return PAE_OK;
    case PAE_Q_SPLITS:
      *value = (long long)P->qkv.splits | ((long long)P->o.splits << 8) | ((long long)P->gu.splits << 16) |
               ((long long)P->down.splits << 24);
      return PAE_OK;
    case PAE_Q_TOKEN_TILE: *value = P->qkv.tn; return PAE_OK;
    case PAE_Q_ATTN_SPLITS: *value = P->attn.splits; return PAE_OK;
    case PAE_Q_PERSISTENT: *value = use_persist(ctx, P) ? 1 : 0; return PAE_OK;
    case PAE_Q_FUSED_NORM: *value = P->fuse_norm ? 1 : P->factored ? 2 : 0; return PAE_OK;
    case PAE_Q_DATAFLOW: *value = use_flow(ctx, P) ? P->fa.C : 0; return PAE_OK;
    case PAE_Q_ATTN_CHUNK: *value = ctx->act_bf16 ? P->attn.chunk : 0; return PAE_OK;
    default: return fail(ctx, PAE_ERR_ARG, "unknown query %d", what);
  }
}

pae_status pae_plan_query(const pae_config* cfg, int what, int batch, long long* value) {
  if (!cfg || !value) return fail(nullptr, PAE_ERR_ARG, "null argument");
  pae_status st = validate_config(cfg);
  if (st != PAE_OK) return st;
  if (batch < 1 || batch > cfg->max_batch) return fail(nullptr, PAE_ERR_ARG, "batch %d out of range", batch);
  if (what != PAE_Q_SPLITS && what != PAE_Q_TOKEN_TILE && what != PAE_Q_ATTN_SPLITS && what != PAE_Q_FUSED_NORM &&
      what != PAE_Q_ATTN_CHUNK)
    return fail(nullptr, PAE_ERR_ARG, "query %d needs a context", what);
  *value = 0;
  if (cfg->dtype == PAE_FP32) return PAE_OK;  // CUDA-core kernels: no tensor-core launch plan
  const Shape s = shape_from_config(cfg);
  const LaunchPlans L = plan_launches(s, batch, cfg->dtype == PAE_W4A16, kDefaultMaxSplitK, false, false);
  switch (what) {
    case PAE_Q_SPLITS:
      *value = (long long)L.qkv.splits | ((long long)L.o.splits << 8) | ((long long)L.gu.splits << 16) |
               ((long long)L.down.splits << 24);
      break;
    case PAE_Q_TOKEN_TILE: *value = L.qkv.tn; break;
    case PAE_Q_ATTN_SPLITS: *value = L.attn.splits; break;
    case PAE_Q_ATTN_CHUNK: *value = L.attn.chunk; break;
    default: *value = L.fuse_norm ? 1 : L.factored ? 2 : 0; break;
  }
  return PAE_OK;
}

pae_status pae_sync(pae_ctx* ctx, pae_stream stream) {
  if (!ctx) return fail(nullptr, PAE_ERR_ARG, "ctx is NULL");
  CK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  CK(cudaGetLastError());
  return check_err_word(ctx);
}

void pae_clear_error(pae_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  // a failed drain stays: the context's memory may still be written by copies
  if (ctx->err_host && *(volatile int*)ctx->err_host != DEV_DRAIN) *(volatile int*)ctx->err_host = 0;
  ctx->last_error.clear();
}

const char* pae_last_error(const pae_ctx* ctx) {
  return ctx ? ctx->last_error.c_str() : g_create_error.c_str();
}

pae_status pae_debug_copy(pae_ctx* ctx, const char* name, void* dst_host, size_t* bytes) {
  if (!ctx || !name || !bytes) return fail(ctx, PAE_ERR_ARG, "null argument");
  const Shape& s = ctx->s;
  const size_t es = ctx->esize;
  const size_t Mmax = (size_t)s.Bmax * s.H;
  const void* src = nullptr;
  size_t n = 0;
  const std::string nm(name);
  if (nm == "x") { src = ctx->x; n = sizeof(float) * Mmax * s.A; }
  else if (nm == "h") { src = ctx->h; n = sizeof(float) * Mmax * s.D; }
  else if (nm == "y") { src = ctx->y; n = Mmax * s.D * es; }
  else if (nm == "q") { src = ctx->q; n = Mmax * s.attn_dim * es; }
  else if (nm == "o") { src = ctx->o; n = Mmax * s.attn_dim * es; }
  else if (nm == "u") { src = ctx->u; n = Mmax * s.F * es; }
  else if (nm == "kcache") { src = ctx->kc; n = (size_t)s.L * s.Bmax * s.Hkv * s.Ptot * s.d * es; }
  else if (nm == "vcache") { src = ctx->vc; n = (size_t)s.L * s.Bmax * s.Hkv * s.Ptot * s.d * es; }
  else if (nm == "tables") { src = ctx->tables; n = sizeof(float) * (size_t)std::max(ctx->K, 1) * s.table_rows; }
  else if (nm == "dt") { src = ctx->dt; n = sizeof(float) * std::max(ctx->K, 1); }
  else if (nm == "lens") { src = ctx->lens_dev; n = sizeof(int) * s.Bmax; }
  else return fail(ctx, PAE_ERR_ARG, "unknown buffer '%s'", name);
  if (!dst_host) { *bytes = n; return PAE_OK; }
  if (*bytes < n) return fail(ctx, PAE_ERR_ARG, "buffer '%s' needs %zu bytes", name, n);
  CK(cudaDeviceSynchronize());
  CK(cudaMemcpy(dst_host, src, n, cudaMemcpyDeviceToHost));
  *bytes = n;
  return PAE_OK;
}

void pae_destroy(pae_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  free_all(ctx);
  delete ctx;
}

}  // extern "C"
