// Small-batch denoise loop as one launch of thread-block clusters (the
// "dataflow loop", for batch * chunk <= 64 action tokens).
//
// At batch 1 the expert's projections are weight streams with 50 tokens each,
// and the graph of ~126 dependent kernels per Euler step spends its time in
// launch, set-up and drain.  Here one cooperative launch runs all Euler steps
// of a call; inside it every stage of a layer
//   Q  [q | k | v] = norm(h) W_qkv^T   (q, and k / v into the request's slot)
//   A  GQA attention over [cached prefix | action keys]
//   O  h += gate_a * (o W_o^T)
//   G  u = gelu(norm(h) W_gate^T) * (norm(h) W_up^T)
//   D  h += gate_m * (u W_down^T)
// waits only for the data it reads, through per-unit counters in global
// memory (release / acquire), never for a grid-wide barrier.
//
// Work split.  The grid is NC clusters of C CTAs (one CTA per SM).
//  * QKV and gate/up (K = width) are cut into 128-row units, and one CTA
//    multiplies a unit over the whole K range (tcgen05, weights as the MMA's
//    M side, tokens as N = 64, fp32 accumulators in TMEM): no partial sum
//    leaves the CTA.  A gate/up unit holds 64 gate rows and the 64 up rows of
//    the same features (two 64-row weight boxes per K block), so the unit's
//    own epilogue forms the GeGLU product.
//  * O and down (K = heads x head_dim, and the MLP width) split K over the C
//    ranks of a cluster, one 128-row tile per cluster.  The C partial tiles
//    are summed by a reduce-scatter inside the cluster: rank p stages rows
//    [q R, q R + R) of its partial for rank q and sends them with one bulk
//    copy into q's shared memory (counted in bytes by q's mbarrier); rank q
//    adds the C slices in rank order (bitwise reproducible) and runs the
//    epilogue for its R = 128 / C rows.
//  * Attention: one cluster per (request, KV head, 128 query rows), its ranks
//    taking consecutive 64-key chunks (online softmax); rank p sends its
//    unnormalised output rows (bf16) and their running max and sum (fp32) to
//    the rows' owner, which merges the C partial softmaxes in fp32.
// A receiver tells its peers that its receive area is free (one remote
// mbarrier arrival each) as soon as it is, long before the data is ready, so
// an exchange costs no cluster barrier.  A peer's arrival for the next
// exchange also tells the sender that its previous copies have landed, so
// the staging area is reused only then.
//
// adaRMSNorm.  y = h rstd (1 + scale) + shift is not formed: the producer of
// h writes bf16(h (1 + scale)) and per-row sums of squares once, and the
// consumer's epilogue applies rstd after the contraction and adds the shift
// term W shift from a table built with the timestep tables.  The same value
// as W y, with no re-normalisation of fp32 h in every unit.
//
// Weights never depend on activations: warp 0 streams this CTA's weight
// blocks into a ring of shared memory in schedule order and prefetches the
// same blocks of the next layer into L2, so HBM keeps streaming while the
// dependency chain runs.  Warp 1 issues the MMAs; warps 2-5 do the rest
// (token operands by TMA, TMEM reads, exchanges, epilogues, the attention
// softmax and the per-token transition between Euler steps).
//
// Every wait is bounded (%globaltimer).  A wait that runs out records
// PAE_ERR_TIMEOUT and sets a launch-wide abort flag that every other wait
// watches.  Before exit every CTA drains its copies, MMAs and any exchange
// still open, and meets its cluster once more (a hardware cluster barrier
// that all threads reach on every path), so no CTA leaves while a peer may
// still write its shared memory.
#include "epilogue.cuh"
#include "launch.cuh"

namespace pae {

namespace {

constexpr int kFThreads = 192;   // warp 0 weights, warp 1 MMA, warps 2-5 compute
constexpr int kFCompute = 128;
constexpr int kFRing = 5;                // bf16 weight ring depth (W4A16: 4 slots + the packed ring)
constexpr int kFRawRing = 4;             // packed int4 blocks [128 rows][32 bytes] in flight (W4A16)
constexpr uint32_t kFRawBlk = 4096;
constexpr uint32_t kFBlk = 16384;        // [128 rows][64] bf16 weight block
constexpr uint32_t kFWork = 128 * 1024;  // operands, epilogue tiles, attention tiles, receive areas
constexpr uint32_t kFMisc = 4096;
constexpr uint32_t kFSmem = kFRing * kFBlk + kFWork + kFMisc + 1024;
constexpr uint32_t kFOp = 0;             // token operand [kb][64 tokens][64] bf16
constexpr uint32_t kFRx = 64 * 1024;     // split-K receive area [C][R rows][Mp tokens] fp32 (<= 32 KB)
constexpr uint32_t kFStg = 96 * 1024;    // split-K rows staged by owner [C][R][Mp] fp32 (<= 32 KB)
constexpr uint32_t kFAStg = 64 * 1024;   // attention rows staged by owner [C][R][d] bf16 (<= 64 KB)
constexpr uint32_t kFTmem = 512;
constexpr uint32_t kColS = 128;          // attention scores (P over their first 32 columns)
constexpr uint32_t kColO = 256;          // attention output
constexpr int CKF = 64;                  // keys per attention chunk
constexpr long long kFDrain = 4000000000LL;
constexpr long long kFExitWait = 2000000LL;  // an exchange left open by an abort, at exit

enum : int { ST_Q = 0, ST_O = 1, ST_G = 2, ST_D = 3 };

// Stage timestamps for performance analysis, compiled in only with
// -DPAE_FLOW_TRACE: compute thread 0 (events 0-6 of a stage, 40-47 of
// attention) and the MMA thread (events 7-9 of a stage) of every CTA record
// %globaltimer at fixed points of one layer (layer 1 of the first step of a
// launch) into g_flow_trace[cta][event]; pae_flow_trace_read copies them out.
#ifdef PAE_FLOW_TRACE
constexpr int kTraceEv = 48;
__device__ unsigned long long g_flow_trace[256 * kTraceEv];
#define FTRACE(c, on, ev)                                                                  \
  do {                                                                                     \
    if ((on) && (c).ct == 0) g_flow_trace[(c).cta * kTraceEv + (ev)] = globaltimer_ns(); \
  } while (0)
#else
#define FTRACE(c, on, ev) \
  do {                    \
  } while (0)
#endif

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_u32(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global_f() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void csync() {
  __syncwarp();
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// AND over the 128 compute threads.
__device__ __forceinline__ bool cand(bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void hw_cluster_sync() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap* tm, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(tm)),
               "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  return (uint32_t)__bfloat16_as_ushort(f2bf(a)) | ((uint32_t)__bfloat16_as_ushort(f2bf(b)) << 16);
}
__device__ __forceinline__ void st_shared_f4(uint32_t addr, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Stores into another CTA's shared memory whose completion is counted (in
// bytes) by an mbarrier of that CTA.
__device__ __forceinline__ void st_async_f2(uint32_t addr, float a, float b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr), "f"(a),
               "f"(b), "r"(rbar)
               : "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory into another CTA's,
// counted (in bytes) by that CTA's mbarrier (both cluster addresses).
__device__ __forceinline__ void bulk_push(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t rbar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src), "r"(bytes), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

struct FMaps {
  const CUtensorMap* w[4];   // weights: Q, O, D with 128-row boxes; G with 64-row boxes
  const CUtensorMap* x[4];   // token operands: y (QKV), o, y (gate/up), u
  const CUtensorMap *q, *k, *v;
};

struct FC {
  const Shape* s;
  const FlowArgs* a;
  FMaps mp;
  uint8_t* ring;
  uint8_t* work;
  uint64_t* rfull;     // [kFRing] bf16 weight block in slot ready for the MMAs
  uint64_t* rempty;    // [kFRing]
  uint64_t* raw_full;  // [kFRawRing] packed int4 block landed (W4A16)
  uint8_t* raw;        // packed int4 ring (W4A16)
  int nring;           // ring depth in use (kFRing, or kFRing - 1 with the int4 ring)
  uint64_t* op_full;   // [4] token operand groups of a projection stage landed
  uint64_t* acc_full;  // [2] split-K accumulator slot ready
  uint64_t* acc_empty; // [2] split-K accumulator slot read out
  uint64_t* acc_all;   // every whole-K unit of a stage accumulated
  uint64_t* kv_full;   // attention q / K / V chunk landed
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_full;
  uint64_t* rx;        // exchange: this CTA's receive area filled (1 arrival + bytes)
  uint64_t* rdy;       // exchange: every peer's receive area free (C - 1 arrivals)
  uint64_t* drain;
  float* s_rstd;       // [64]
  float* s_tmp;        // [512]
  float* s_st;         // [C][R][2] attention (max, sum) received for this rank's rows
  int* s_len;          // [64] prefix length of every request (fixed during a launch)
  volatile int* s_abort;
  volatile int* s_flag;
  uint32_t tmem;
  int cta, ncta, cl, rank, ct;  // ct: compute-thread index 0..127
};

__device__ __forceinline__ unsigned* abort_word(const FlowArgs& a) { return a.ctr + kFlowCtrWords - 1; }

// Launch-wide abort: record the error, stop this CTA's roles, tell all CTAs.
__device__ void raise_abort(const FC& c) {
  *c.s_abort = 1;
  atomicExch(reinterpret_cast<int*>(abort_word(*c.a)), 1);
  set_error(c.a->err, DEV_TIMEOUT);
}

// Bounded mbarrier wait (acquire at cluster scope, which also covers data
// that other CTAs of the cluster stored) that gives up once the launch is
// aborting.
__device__ bool fwait(const FC& c, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  const volatile unsigned* ab = abort_word(*c.a);
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*c.s_abort || *ab) {
      *c.s_abort = 1;
      return false;
    }
    if ((long long)(globaltimer_ns() - t0) > c.a->err.wait_ns) {
      raise_abort(c);
      return false;
    }
  }
}

// One compute thread waits on the mbarrier, the others on the CTA barrier
// that follows (it orders their later reads after that thread's acquire):
// 128 threads polling one mbarrier would take shared-memory bandwidth from
// the copies landing in this CTA.  Returns false once the launch is aborting.
__device__ bool cwait(const FC& c, uint64_t* bar, uint32_t parity) {
  bool ok = true;
  if (c.ct == 0) ok = fwait(c, bar, parity);
  return cand(ok);
}

// Bounded wait until a global counter reaches `target` (acquire).
__device__ bool wait_ctr(const FC& c, const unsigned* p, unsigned target) {
  if (ld_acquire_u32(p) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  const volatile unsigned* ab = abort_word(*c.a);
  while (true) {
    if (ld_acquire_u32(p) >= target) return true;
    if (*c.s_abort || *ab) {
      *c.s_abort = 1;
      return false;
    }
    if ((long long)(globaltimer_ns() - t0) > c.a->err.wait_ns) {
      raise_abort(c);
      return false;
    }
  }
}

// Bounded wait by one whole warp until the counters p[0..n) all reach
// `target`: lane i polls p[i], p[i + 32], ..., so every load is in flight at
// once (one round trip instead of n).  Warp-uniform result; the closing
// __syncwarp orders every lane's acquire before what lane 0 does next.
__device__ bool wait_ctrs(const FC& c, const unsigned* p, int n, unsigned target) {
  const int lane = threadIdx.x & 31;
  auto done = [&]() {
    bool d = true;
    for (int i = lane; i < n; i += 32) d = ld_acquire_u32(p + i) >= target && d;
    return __all_sync(0xffffffffu, d);
  };
  const unsigned long long t0 = globaltimer_ns();
  const volatile unsigned* ab = abort_word(*c.a);
  while (!done()) {
    int stop = 0;  // 1: the launch is aborting, 2: this wait ran out
    if (lane == 0) {
      if (*c.s_abort || *ab) stop = 1;
      else if ((long long)(globaltimer_ns() - t0) > c.a->err.wait_ns) stop = 2;
    }
    stop = __shfl_sync(0xffffffffu, stop, 0);
    if (stop) {
      if (lane == 0) {
        if (stop == 2) raise_abort(c);
        else *c.s_abort = 1;
      }
      __syncwarp();
      return false;
    }
  }
  __syncwarp();
  return true;
}

// Every compute thread's global writes, then one release increment of `p`.
__device__ void publish(const FC& c, unsigned* p) {
  __threadfence();
  csync();
  if (c.ct == 0) red_release_u32(p, 1u);
}

// ------------------------------------------------------------ exchanges
// An exchange moves data between the C ranks of a cluster into each rank's
// receive area.  `xn` counts this CTA's exchanges; every rank of a cluster
// takes part in the same exchanges in the same order, so the mbarrier phases
// agree.
//  open:  the receive area is free: arm rx for `bytes` from the peers, then
//         one remote arrival on every peer's rdy (release: everything this
//         CTA did with the area before is ordered before the peers' stores).
//  ready: every peer's area is free (rdy complete), so stores may start.
//  wait:  every peer's bytes landed (rx complete) and this CTA's own slice,
//         written with plain stores, is visible to all compute threads.
__device__ void xchg_open(const FC& c, uint32_t bytes) {
  const int C = c.a->C;
  if (C == 1 || c.ct != 0 || *c.s_abort) return;
  mbar_arrive_expect_tx(c.rx, bytes);
  for (int q = 1; q < C; ++q) {
    const uint32_t peer = (uint32_t)((c.rank + q) % C);
    mbar_arrive_remote(map_cluster(smem_u32(c.rdy), peer));
  }
}
__device__ bool xchg_ready(const FC& c, int xn) {
  if (c.a->C == 1) return true;
  bool ok = true;
  if (c.ct == 0) ok = !*c.s_abort && fwait(c, c.rdy, (uint32_t)xn & 1u);
  if (!cand(ok)) return false;
  return mbar_try_wait_cl(c.rdy, (uint32_t)xn & 1u);  // each thread's own acquire (complete by now)
}
__device__ bool xchg_wait(const FC& c, int xn) {
  csync();  // own slice stored
  if (c.a->C == 1) return true;
  bool ok = true;
  if (c.ct == 0) ok = !*c.s_abort && fwait(c, c.rx, (uint32_t)xn & 1u);
  if (!cand(ok)) return false;
  return mbar_try_wait_cl(c.rx, (uint32_t)xn & 1u);
}

// ------------------------------------------------------------ schedule
// Projection stage geometry: units (Q, G: 128-row whole-K units; O, D:
// 128-row tiles split over the cluster), K blocks per unit or per rank, and
// weight rows per layer.
struct StageG {
  int units, kb, wrows;
  bool whole;
};
__device__ __forceinline__ StageG stage_geo(const Shape& s, const FlowArgs& a, int st) {
  switch (st) {
    case ST_Q: return StageG{a.q_units, a.kb_q, s.qkv_rows, true};
    case ST_O: return StageG{a.o_tiles, a.kb_o, s.D, false};
    case ST_G: return StageG{a.g_units, a.kb_g, 2 * s.F, true};
    default: return StageG{a.d_tiles, a.kb_d, s.D, false};
  }
}
// Units owned by this CTA (whole-K: unit i runs on CTA (base + i) mod ncta)
// or by its cluster (tiles: tile t runs on cluster (base + t) mod NC): the
// count, and the first one in `first`; the others follow every n.
__device__ __forceinline__ int owned(const FC& c, int st, const StageG& g, int& first) {
  const FlowArgs& a = *c.a;
  const bool w = g.whole;
  const int n = w ? c.ncta : a.NC, me = w ? c.cta : c.cl;
  const int base = st == ST_Q ? a.q_base : st == ST_O ? a.o_base : st == ST_G ? a.g_base : a.d_base;
  first = ((me - base) % n + n) % n;
  return first < g.units ? (g.units - first + n - 1) / n : 0;
}
__device__ __forceinline__ int unit_step(const FC& c, const StageG& g) { return g.whole ? c.ncta : c.a->NC; }
// Stored weight rows of unit / tile t in layer l: the first box's first row,
// and the second 64-row half's (gate/up: the up rows of the same features).
__device__ __forceinline__ void unit_rows(const Shape& s, int st, const StageG& g, int l, int t, int& r0, int& r1) {
  if (st == ST_G) {
    r0 = l * g.wrows + 256 * (t >> 1) + 64 * (t & 1);
    r1 = r0 + 128;
  } else {
    r0 = l * g.wrows + 128 * t;
    r1 = r0 + 64;
  }
}

// Attention unit of cluster cl: (request b, KV head g, 128-row query tile
// qt); this rank's keys [start, end) of the slot.
struct AttU {
  bool has;
  int b, g, bg, qt, start, end, nch;
};
__device__ __forceinline__ AttU att_unit(const Shape& s, const FlowArgs& a, int cl, int rank) {
  AttU u{};
  const int unit = ((cl - a.a_base) % a.NC + a.NC) % a.NC;
  u.has = unit < a.a_units;
  if (!u.has) return u;
  u.bg = unit / a.a_qtiles;
  u.qt = unit - u.bg * a.a_qtiles;
  u.b = u.bg / s.Hkv;
  u.g = u.bg - u.b * s.Hkv;
  const int n_valid = __ldg(a.lens + u.b) + s.H;  // set before the launch, fixed during it
  u.start = rank * a.a_kps;
  u.end = min(n_valid, u.start + a.a_kps);
  u.nch = u.end > u.start ? (u.end - u.start + CKF - 1) / CKF : 0;
  return u;
}

// Counter words.
__device__ __forceinline__ unsigned* c_tr(const FlowArgs& a) { return a.ctr + 0; }
__device__ __forceinline__ unsigned* c_qkv(const FlowArgs& a) { return a.ctr + 1; }
__device__ __forceinline__ unsigned* c_att(const FlowArgs& a) { return a.ctr + 2; }
__device__ __forceinline__ unsigned* c_y(const FlowArgs& a, int t) { return a.ctr + 3 + t; }
__device__ __forceinline__ unsigned* c_ho(const FlowArgs& a, int t) { return a.ctr + 3 + a.d_tiles + t; }
__device__ __forceinline__ unsigned* c_u(const FlowArgs& a, int j) { return a.ctr + 3 + a.d_tiles + a.o_tiles + j; }

// Operand groups: the K blocks of a stage's token operand arrive in up to 4
// groups, each on its own mbarrier, so the first MMAs start before the last
// blocks land.  Group gi holds blocks [gi gsz, min(kb, (gi + 1) gsz)).
__device__ __forceinline__ int op_gsz(int kb) { return (kb + 3) / 4; }

// ------------------------------------------------------------ weight producer
// Weight block n of this CTA's schedule (per step, layer, stage, unit, K
// block): which matrix, its K offset (elements), the rows of its two 64-row
// halves, and the row offset of the same block in the next layer (or layer 0
// of the next step; `last`: none).
struct Blk {
  int st, kofs, row0, row1, dnext;
  bool last;
};
__device__ __forceinline__ int blocks_per_layer(const FC& c) {
  int n = 0;
  for (int st = 0; st < 4; ++st) {
    const StageG g = stage_geo(*c.s, *c.a, st);
    int first;
    n += owned(c, st, g, first) * g.kb;
  }
  return n;
}
__device__ bool block_at(const FC& c, int nbl, int n, Blk& b) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  if (nbl == 0) return false;
  const int kl = n / nbl;
  if (kl >= (a.k_end - a.k_begin) * s.L) return false;
  int r = n - kl * nbl;
  const int l = kl % s.L;
  for (int st = 0; st < 4; ++st) {
    const StageG g = stage_geo(s, a, st);
    int first;
    const int cnt = owned(c, st, g, first) * g.kb;
    if (r < cnt) {
      const int item = r / g.kb, i = r - item * g.kb;
      b.st = st;
      b.kofs = (g.whole ? i : c.rank * g.kb + i) * 64;
      unit_rows(s, st, g, l, first + item * unit_step(c, g), b.row0, b.row1);
      b.last = kl + 1 >= (a.k_end - a.k_begin) * s.L;
      b.dnext = l + 1 < s.L ? g.wrows : -(s.L - 1) * g.wrows;
      return true;
    }
    r -= cnt;
  }
  return false;
}

// Packed int4 weights -> bf16 code * group scale, rounded once (to nearest
// even): two codes per call from one 32-bit word whose nibbles were permuted
// at create time so that (w >> 4i) & 0x000F000F holds the pair (2i, 2i + 1).
// (n ^ 8) | 0x4300 is the bf16 of 128 + (code + 8); subtracting 136 is exact.
__device__ __forceinline__ uint32_t dq_pair(uint32_t w, int i, __nv_bfloat162 sc) {
  const uint32_t t = (((w >> (4 * i)) & 0x000F000Fu) ^ 0x00080008u) | 0x43004300u;
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&t);
  const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
  v = __hmul2(__hsub2(v, off), sc);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Warp 0.  bf16 weights: lane 0 streams this CTA's weight blocks (16 KB: one
// 128-row box, or for gate/up two 64-row boxes) into the ring in schedule
// order.  int4 weights: lane 0 keeps kFRawRing packed blocks (4 KB) in
// flight; all 32 lanes turn each landed block into a bf16 block of the ring
// (4 rows per lane, 128-byte swizzled like a TMA tile).  Either way each load
// also prefetches the same block of the next layer into L2, so HBM streams
// one layer ahead of the dependency chain.
__device__ void producer_warp(const FC& c) {
  const FlowArgs& a = *c.a;
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_first();  // a block is used once per step
  const int nbl = blocks_per_layer(c);
  const int R = c.nring;
  int n = 0;
  bool ok = true;
  if (!a.w4) {
    if (lane == 0) {
      Blk b;
      for (; block_at(c, nbl, n, b); ++n) {
        const int slot = n % R;
        if (n >= R && !fwait(c, &c.rempty[slot], ((n / R) & 1) ^ 1)) {
          ok = false;
          break;
        }
        uint8_t* dst = c.ring + (size_t)slot * kFBlk;
        const CUtensorMap* tm = c.mp.w[b.st];
        mbar_arrive_expect_tx(&c.rfull[slot], kFBlk);
        if (b.st == ST_G) {
          tma_load_2d_hint(dst, tm, b.kofs, b.row0, &c.rfull[slot], pol);
          tma_load_2d_hint(dst + kFBlk / 2, tm, b.kofs, b.row1, &c.rfull[slot], pol);
          if (!b.last) {
            tma_prefetch_l2(tm, b.kofs, b.row0 + b.dnext);
            tma_prefetch_l2(tm, b.kofs, b.row1 + b.dnext);
          }
        } else {
          tma_load_2d_hint(dst, tm, b.kofs, b.row0, &c.rfull[slot], pol);
          if (!b.last) tma_prefetch_l2(tm, b.kofs, b.row0 + b.dnext);
        }
      }
      // copies still in flight land before the CTA exits
      for (int j = n > R ? n - R : 0; j < n; ++j)
        if (!mbar_wait(&c.rfull[j % R], (j / R) & 1, kFDrain)) set_error(a.err, DEV_DRAIN);
    }
    __syncwarp();
    return;
  }
  // ---- int4: packed blocks in flight, dequantised by the whole warp
  int issued = 0;
  auto issue = [&](int m) -> bool {
    Blk b;
    if (!block_at(c, nbl, m, b)) return false;
    const int rs = m % kFRawRing;
    uint8_t* dst = c.raw + (size_t)rs * kFRawBlk;
    const CUtensorMap* tm = c.mp.w[b.st];
    mbar_arrive_expect_tx(&c.raw_full[rs], kFRawBlk);
    if (b.st == ST_G) {
      tma_load_2d_hint(dst, tm, b.kofs / 2, b.row0, &c.raw_full[rs], pol);
      tma_load_2d_hint(dst + kFRawBlk / 2, tm, b.kofs / 2, b.row1, &c.raw_full[rs], pol);
      if (!b.last) {
        tma_prefetch_l2(tm, b.kofs / 2, b.row0 + b.dnext);
        tma_prefetch_l2(tm, b.kofs / 2, b.row1 + b.dnext);
      }
    } else {
      tma_load_2d_hint(dst, tm, b.kofs / 2, b.row0, &c.raw_full[rs], pol);
      if (!b.last) tma_prefetch_l2(tm, b.kofs / 2, b.row0 + b.dnext);
    }
    return true;
  };
  if (lane == 0)
    while (issued < kFRawRing && issue(issued)) ++issued;
  issued = __shfl_sync(0xffffffffu, issued, 0);
  Blk b;
  for (; ok && block_at(c, nbl, n, b); ++n) {
    const int rs = n % kFRawRing, slot = n % R;
    bool w = fwait(c, &c.raw_full[rs], (n / kFRawRing) & 1);
    if (w && n >= R) w = fwait(c, &c.rempty[slot], ((n / R) & 1) ^ 1);
    if (!__all_sync(0xffffffffu, w)) {
      ok = false;
      break;
    }
    // rows lane, lane + 32, lane + 64, lane + 96 of the block; rows 64.. are
    // the second box (gate/up: the up rows)
    const StageG g = stage_geo(*c.s, a, b.st);
    const int K = g.whole ? g.kb * 64 : g.kb * 64 * a.C;  // the matrix's K
    const int gpr = K / 128, grp = b.kofs / 128;
    const uint8_t* rb = c.raw + (size_t)rs * kFRawBlk;
    const uint32_t ab = smem_u32(c.ring + (size_t)slot * kFBlk);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = lane + 32 * q;
      const int srow = r < 64 ? b.row0 + r : b.row1 + (r - 64);
      const bf16 sv = a.wsc[b.st][(size_t)srow * gpr + grp];
      const __nv_bfloat162 sc = __halves2bfloat162(sv, sv);
      const uint4 w0 = *reinterpret_cast<const uint4*>(rb + r * 32);
      const uint4 w1 = *reinterpret_cast<const uint4*>(rb + r * 32 + 16);
      const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint32_t addr = ab + (uint32_t)r * 128u + (((uint32_t)cc ^ (uint32_t)(r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dq_pair(words[cc], 0, sc)),
                     "r"(dq_pair(words[cc], 1, sc)), "r"(dq_pair(words[cc], 2, sc)), "r"(dq_pair(words[cc], 3, sc))
                     : "memory");
      }
    }
    fence_proxy_async_smem();  // the tensor cores read what the warp just wrote
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&c.rfull[slot]);
      if (issue(issued)) ++issued;  // the raw slot of block n is free now
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
  }
  if (!ok && !*c.s_abort) raise_abort(c);
  // packed copies still in flight land before the CTA exits
  if (lane == 0)
    for (int j = issued > kFRawRing ? issued - kFRawRing : 0; j < issued; ++j)
      if (!mbar_wait(&c.raw_full[j % kFRawRing], (j / kFRawRing) & 1, kFDrain)) set_error(a.err, DEV_DRAIN);
  __syncwarp();
}

// ------------------------------------------------------------ MMA issuer
// Warp 1, lane 0.  Whole-K stage: unit j of this CTA accumulates
// D[128 rows][64 tokens] in TMEM columns 64 j over all K blocks, one commit
// for the stage.  Split-K stage: tile item it accumulates this rank's K
// blocks in slot it % 2 (columns 0 / 64), one commit per item.  Attention
// chunk: S = Q K^T (M = 128 query rows, N = 64 keys), then O += P V with P
// read from TMEM and V MN-major from shared memory.
__device__ void mma_loop(const FC& c) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const int d = s.d;
  const uint32_t idg = idesc_bf16(128, 64);
  const uint32_t ids = idesc_bf16(128, CKF);
  const uint32_t ido = idesc_bf16(128, d, 0, 1);
  const uint32_t work = smem_u32(c.work), ring = smem_u32(c.ring);
  const uint32_t qbytes = 128u * d * 2u, kvbytes = (uint32_t)CKF * d * 2u;
  const AttU au = att_unit(s, a, c.cl, c.rank);
  int n = 0, it = 0, ac = 0;
  int opn[4] = {0, 0, 0, 0};
  bool ok = true;
  for (int k = a.k_begin; ok && k < a.k_end; ++k)
    for (int l = 0; ok && l < s.L; ++l)
      for (int st5 = 0; ok && st5 < 5; ++st5) {
        if (st5 == 1) {
          if (!au.has) continue;
          for (int ch = 0; ch < au.nch; ++ch, ++ac) {
            if (!fwait(c, c.kv_full, ac & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int k16 = 0; k16 < d / 16; ++k16) {
              const uint32_t x = (uint32_t)k16 >> 2, w = ((uint32_t)k16 & 3u) * 32u;
              umma_bf16(c.tmem + kColS, sw128_desc(work + x * 128u * 128u + w, 16, 1024),
                        sw128_desc(work + qbytes + x * (uint32_t)CKF * 128u + w, 16, 1024), ids, k16 > 0 ? 1u : 0u);
            }
            umma_commit(c.s_full);
            if (!fwait(c, c.p_full, ac & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t vd = sw128_desc(work + qbytes + kvbytes, CKF * 128, 1024);
            for (int k16 = 0; k16 < CKF / 16; ++k16)
              umma_bf16_tmem_a(c.tmem + kColO, c.tmem + kColS + (uint32_t)k16 * 8u, desc_add(vd, k16 * 16u * 128u), ido,
                               (ch > 0 || k16 > 0) ? 1u : 0u);
            umma_commit(c.o_full);
          }
          continue;
        }
        const int st = st5 == 0 ? ST_Q : st5 - 1;
        const StageG g = stage_geo(s, a, st);
        int first;
        const int nu = owned(c, st, g, first);
        if (nu == 0) continue;
        const int gsz = op_gsz(g.kb);
#ifdef PAE_FLOW_TRACE
        const bool trm = k == a.k_begin && l == 1;
#endif
        for (int j = 0; ok && j < nu; ++j) {
          uint32_t col;
          if (g.whole) {
            col = 64u * (uint32_t)j;
          } else {
            const int slot = it & 1;
            if (it >= 2 && !fwait(c, &c.acc_empty[slot], ((it >> 1) & 1) ^ 1)) {
              ok = false;
              break;
            }
            col = 64u * (uint32_t)slot;
          }
          tc_fence_after();
          for (int i = 0; i < g.kb; ++i, ++n) {
            if (j == 0 && i % gsz == 0) {
              const int gi = i / gsz;
              if (!fwait(c, &c.op_full[gi], (uint32_t)opn[gi] & 1u)) {
                ok = false;
                break;
              }
              ++opn[gi];
#ifdef PAE_FLOW_TRACE
              if (trm && gi == 0) g_flow_trace[c.cta * kTraceEv + st * 10 + 7] = globaltimer_ns();
#endif
            }
            const int rs = n % c.nring;
            if (!fwait(c, &c.rfull[rs], (n / c.nring) & 1)) {
              ok = false;
              break;
            }
#ifdef PAE_FLOW_TRACE
            if (trm && j == 0 && i == 0) g_flow_trace[c.cta * kTraceEv + st * 10 + 8] = globaltimer_ns();
#endif
            tc_fence_after();
            const uint32_t sa = ring + (uint32_t)rs * kFBlk, sb = work + kFOp + (uint32_t)i * 8192u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(c.tmem + col, sw128_desc(sa + kk * 32, 16, 1024), sw128_desc(sb + kk * 32, 16, 1024), idg,
                        (i > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&c.rempty[rs]);
          }
          if (!ok) break;
          if (!g.whole) {
            umma_commit(&c.acc_full[it & 1]);
            ++it;
          }
        }
        if (!ok) break;
        if (g.whole) umma_commit(c.acc_all);
#ifdef PAE_FLOW_TRACE
        if (trm) g_flow_trace[c.cta * kTraceEv + st * 10 + 9] = globaltimer_ns();
#endif
      }
  if (!ok && !*c.s_abort) raise_abort(c);
  // every MMA this thread issued must finish before TMEM is freed
  umma_commit(c.drain);
  if (!mbar_wait(c.drain, 0, kFDrain)) set_error(a.err, DEV_DRAIN);
}

// ------------------------------------------------------------ compute side
__device__ __forceinline__ float4 ldcg_f4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ldg_f4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void f4_to(float* v, float4 a, float4 b) {
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf2(v[0], v[1]), pack_bf2(v[2], v[3]), pack_bf2(v[4], v[5]), pack_bf2(v[6], v[7]));
}

// Deterministic sum over the 128 compute threads (fixed tree).
__device__ float csum(const FC& c, float v) {
  v = warp_sum(v);
  const int lane = c.ct & 31, w = c.ct >> 5;
  csync();
  if (lane == 0) c.s_tmp[w] = v;
  csync();
  return ((c.s_tmp[0] + c.s_tmp[1]) + c.s_tmp[2]) + c.s_tmp[3];
}

// Epilogue of the QKV projection for 8 stored rows f0.. of token m: rstd and
// the shift term, then q (head-major) or this step's key / value into the
// request's slot at position len + i; rotated heads store their 4 pairs on
// channels i0.. and i0 + d/2.., turned by the (cos, sin) values cs[0..4).
__device__ void epi_q(const FC& c, int l, int m, int len, int f0, const float* acc, const float* bv,
                      const float2* cs) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const float rs = c.s_rstd[m];
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = fmaf(rs, acc[i], bv[i]);
  const int b = m / s.H, tt = m - b * s.H;
  const int qd = s.Hq * s.d, kvd = s.Hkv * s.d;
  bf16* base;
  int j;
  if (f0 < qd) {
    const int head = f0 / s.d;
    j = f0 - head * s.d;
    base = a.q + ((size_t)(b * s.Hq + head) * s.H + tt) * s.d;
  } else {
    const bool is_v = f0 >= qd + kvd;
    const int fk = f0 - qd - (is_v ? kvd : 0);
    const int g = fk / s.d;
    j = fk - g * s.d;
    base = (is_v ? a.vc : a.kc) + (((size_t)(l * s.Bmax + b) * s.Hkv + g) * s.Ptot + len + tt) * s.d;
  }
  if (cs) {
    const int i0 = j >> 1;
    float lo[4], hi[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 t = cs[u];
      const float x = v[2 * u], y = v[2 * u + 1];
      lo[u] = x * t.x - y * t.y;
      hi[u] = y * t.x + x * t.y;
    }
    *reinterpret_cast<uint2*>(base + i0) = make_uint2(pack_bf2(lo[0], lo[1]), pack_bf2(lo[2], lo[3]));
    *reinterpret_cast<uint2*>(base + i0 + (s.d >> 1)) = make_uint2(pack_bf2(hi[0], hi[1]), pack_bf2(hi[2], hi[3]));
  } else {
    *reinterpret_cast<uint4*>(base + j) = pack8(v);
  }
}

// Epilogue inputs of one reducing thread (token m, 8 rows from f0), read
// while the exchange is in flight: the residual stream, gate and next norm
// scale (O, down).
struct EpiIn {
  float b[8];  // gate
  float h[8];  // residual stream
  float sc[8]; // next norm's scale (unused without a next norm)
};

// Gated residual for 8 features f0.. of token m: h += gate * acc, then (when
// `has_next`) the next norm's operand bf16(h (1 + scale)) and the sum of the 8
// squares of h.
__device__ float epi_resid(const FC& c, int m, int f0, const float* acc, const EpiIn& in, bool has_next,
                           bf16* ydst) {
  const Shape& s = *c.s;
  float* hp = c.a->h + (size_t)m * s.D + f0;
  float hv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) hv[i] = fmaf(in.b[i], acc[i], in.h[i]);
  reinterpret_cast<float4*>(hp)[0] = make_float4(hv[0], hv[1], hv[2], hv[3]);
  reinterpret_cast<float4*>(hp)[1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
  float ss = 0.f;
  if (has_next) {
    float yv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      yv[i] = hv[i] * (1.f + in.sc[i]);
      ss = fmaf(hv[i], hv[i], ss);
    }
    *reinterpret_cast<uint4*>(ydst + (size_t)m * s.D + f0) = pack8(yv);
  }
  return ss;
}

// rstd per token for the QKV / gate-up norm from the producers' sums of
// squares ss[slot][64]: thread (4 tokens, slot group) sums every 8th slot with
// all its loads in flight, then the 8 group sums per token are added in a
// fixed order.
__device__ void compute_rstd(const FC& c, const float* ss, int nslots) {
  const Shape& s = *c.s;
  const int m4 = c.ct & 15, grp = c.ct >> 4;  // 16 x 4 tokens, 8 slot groups
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = grp; s0 < nslots; s0 += 8 * 16) {
    float4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      v[i] = s0 + 8 * i < nslots ? ldcg_f4(ss + (size_t)(s0 + 8 * i) * 64 + 4 * m4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      acc.x += v[i].x;
      acc.y += v[i].y;
      acc.z += v[i].z;
      acc.w += v[i].w;
    }
  }
  *reinterpret_cast<float4*>(c.s_tmp + grp * 64 + 4 * m4) = acc;
  csync();
  if (c.ct < 64) {
    float t = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) t += c.s_tmp[g * 64 + c.ct];
    c.s_rstd[c.ct] = rsqrtf(t / (float)s.D + s.eps);
  }
  csync();
}

// Compute thread 0: the token operand [64 tokens][kb * 64] from column x0,
// in up to 4 groups (8 KB per block).  `opn` counts each group's uses.
__device__ void issue_operand(const FC& c, int st, int x0, int kb, int* opn) {
  fence_proxy_async_global_f();  // written by other CTAs' generic stores, read by TMA
  fence_proxy_async_smem();      // this CTA's generic stores to the area come first
  const int gsz = op_gsz(kb);
  for (int gi = 0; gi * gsz < kb; ++gi) {
    const int b0 = gi * gsz, b1 = min(kb, b0 + gsz);
    mbar_arrive_expect_tx(&c.op_full[gi], (uint32_t)(b1 - b0) * 8192u);
    for (int i = b0; i < b1; ++i)
      tma_load_2d(c.work + kFOp + (size_t)i * 8192, c.mp.x[st], x0 + i * 64, 0, &c.op_full[gi]);
    ++opn[gi];
  }
}

// QKV or gate/up on this CTA: its whole-K units.  The operand is the full
// width, so every producer of it must be done; rstd comes from all their
// sums of squares.  Each unit's accumulator goes through shared memory
// ([64 tokens][128 rows] fp32, in the operand area once the MMAs are done)
// so that a thread's epilogue covers 8 consecutive features of one token.
// `sw` counts this CTA's whole-K stages (the acc_all phase).
__device__ bool whole_stage(const FC& c, int st, int k, int l, int u, int& sw, int* opn) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const StageG g = stage_geo(s, a, st);
  int first;
  const int nu = owned(c, st, g, first);
  if (nu == 0) return true;
  const unsigned uC = (unsigned)a.C;
  const bool tr = k == a.k_begin && l == 1;
  const int tb = st * 10;
  (void)tr;
  (void)tb;
  FTRACE(c, tr, tb + 0);

  // 1. every producer of the operand, then its TMA
  bool ok = true;
  if (c.ct < 32) {
    if (st == ST_Q && l == 0) ok = wait_ctrs(c, c_tr(a), 1, (unsigned)(a.M * (k - a.k_begin + 1)));
    else if (st == ST_Q) ok = wait_ctrs(c, c_y(a, 0), a.d_tiles, uC * (unsigned)u);
    else ok = wait_ctrs(c, c_ho(a, 0), a.o_tiles, uC * (unsigned)(u + 1));
    if (ok && c.ct == 0) issue_operand(c, st, 0, g.kb, opn);
  }
  FTRACE(c, tr, tb + 1);
  if (!cand(ok)) return false;

  // 2. rstd per token from the producers' sums of squares, while the MMAs run
  if (st == ST_G) compute_rstd(c, a.ss_g, a.o_tiles * a.C);
  else if (l > 0) compute_rstd(c, a.ss_q, a.d_tiles * a.C);
  else compute_rstd(c, a.ss_t, 1);
  FTRACE(c, tr, tb + 2);

  // 3. every unit accumulated: the operand area is free from here on
  if (!cwait(c, c.acc_all, (uint32_t)sw & 1u)) return false;
  ++sw;
  tc_fence_after();
  FTRACE(c, tr, tb + 3);

  // 4. per unit: epilogue inputs staged (bias row in s_tmp; for rotated QKV
  //    rows the (cos, sin) of the unit's 64 pairs at every token's position,
  //    [M][64] float2 after the tile), accumulator -> tile, epilogue
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qd = warp & 3, row = qd * 32 + lane;  // TMEM lane = weight row
  const uint32_t tile = smem_u32(c.work);
  const float2* cstage = reinterpret_cast<const float2*>(c.work + 32768);
  const int Mc = (a.M + 15) & ~15;  // accumulator columns read, 16 at a time
  const float* tb_row = st == ST_Q ? a.bias_qkv + ((size_t)k * s.L + l) * s.qkv_rows
                                   : a.bias_gu + ((size_t)k * s.L + l) * 2 * s.F;
  const int rot_rows = (s.Hq + s.Hkv) * s.d;
  for (int j = 0; j < nu; ++j) {
    const int t = first + j * c.ncta;
    if (j > 0) csync();  // the previous unit's epilogue has read the tile and the staged inputs
    int g0 = 0, g1 = 0;
    if (st == ST_G) unit_rows(s, ST_G, g, 0, t, g0, g1);  // gate and up rows within a layer
    c.s_tmp[c.ct] = st == ST_Q ? tb_row[128 * t + c.ct] : tb_row[c.ct < 64 ? g0 + c.ct : g1 + c.ct - 64];
    const bool rot = st == ST_Q && a.rope_cs != nullptr && 128 * t < rot_rows;
    if (rot) {
      float2* cw = reinterpret_cast<float2*>(c.work + 32768);
      for (int idx = c.ct; idx < a.M * 64; idx += kFCompute) {
        const int m = idx >> 6, jj = idx & 63;
        const int b = m / s.H, pos = c.s_len[b] + (m - b * s.H);
        const int i = ((128 * t + 2 * jj) % s.d) >> 1;
        cw[idx] = a.rope_cs[(size_t)pos * (s.d >> 1) + i];
      }
    }
    const uint32_t taddr = c.tmem + ((uint32_t)(qd * 32) << 16) + 64u * (uint32_t)j;
    for (int c0 = 0; c0 < Mc; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + (uint32_t)c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) st_shared_f32(tile + (uint32_t)(((c0 + jj) * 128 + row) * 4), v[jj]);
    }
    tc_fence_before();
    csync();
    if (st == ST_Q) {
      for (int idx = c.ct; idx < a.M * 16; idx += kFCompute) {
        const int m = idx >> 4, r0 = (idx & 15) * 8;
        float acc[8], bv[8];
        const uint32_t ta = tile + (uint32_t)((m * 128 + r0) * 4);
        f4_to(acc, ld_shared_f4(ta), ld_shared_f4(ta + 16));
#pragma unroll
        for (int i = 0; i < 8; ++i) bv[i] = c.s_tmp[r0 + i];
        const int f0 = 128 * t + r0;
        epi_q(c, l, m, c.s_len[m / s.H], f0, acc, bv, rot && f0 < rot_rows ? cstage + m * 64 + r0 / 2 : nullptr);
      }
    } else {
      for (int idx = c.ct; idx < a.M * 8; idx += kFCompute) {
        const int m = idx >> 3, r0 = (idx & 7) * 8;
        float gv[8], uv[8], ov[8];
        const uint32_t ta = tile + (uint32_t)((m * 128 + r0) * 4);
        f4_to(gv, ld_shared_f4(ta), ld_shared_f4(ta + 16));
        f4_to(uv, ld_shared_f4(ta + 256), ld_shared_f4(ta + 272));
        const float rs = c.s_rstd[m];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          ov[i] = gelu_tanh_bf16out(fmaf(rs, gv[i], c.s_tmp[r0 + i])) * fmaf(rs, uv[i], c.s_tmp[64 + r0 + i]);
        *reinterpret_cast<uint4*>(a.u + (size_t)m * s.F + 64 * t + r0) = pack8(ov);
      }
    }
  }
  FTRACE(c, tr, tb + 4);

  // 5. publish every unit (one fence)
  __threadfence();
  csync();
  if (c.ct == 0) {
    if (st == ST_Q) {
      red_release_u32(c_qkv(a), (unsigned)nu);
    } else {
      for (int j = 0; j < nu; ++j) red_release_u32(c_u(a, first + j * c.ncta), 1u);
    }
  }
  FTRACE(c, tr, tb + 5);
  return true;
}

// O or down on this CTA's cluster: its tiles, K split over the ranks.  Per
// tile, rank p's partial row r goes to rank r / R (R = 128 / C rows each),
// which adds the C slices in rank order and applies the gated residual, the
// next norm's operand and its sums of squares.  `it` counts split-K items
// (TMEM slot), `xn` exchanges; `xopen` marks an exchange armed and not yet
// complete (drained at exit after an abort).
__device__ bool split_stage(const FC& c, int st, int k, int l, int u, int& it, int& xn, bool& xopen, int* opn) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const StageG g = stage_geo(s, a, st);
  int first;
  const int nt = owned(c, st, g, first);
  if (nt == 0) return true;  // uniform over the cluster
  const int C = a.C, R = 128 / C, rank = c.rank;
  const int x0 = rank * g.kb * 64, x1 = x0 + g.kb * 64;
  const bool tr = k == a.k_begin && l == 1;
  const int tb = st * 10;
  (void)tr;
  (void)tb;
  FTRACE(c, tr, tb + 0);

  // 1. the producers of this rank's K slice of the operand, then its TMA
  bool ok = true;
  if (c.ct < 32) {
    if (st == ST_O) ok = wait_ctrs(c, c_att(a), 1, (unsigned)a.a_units * (unsigned)C * (unsigned)(u + 1));
    else ok = wait_ctrs(c, c_u(a, x0 / 64), (x1 - 1) / 64 - x0 / 64 + 1, (unsigned)(u + 1));
    if (ok && c.ct == 0) issue_operand(c, st, x0, g.kb, opn);
  }
  FTRACE(c, tr, tb + 1);
  if (!cand(ok)) return false;

  const float* tab = a.tables + (size_t)k * s.table_rows;
  const bool has_next = st == ST_O || (st == ST_D && l + 1 < s.L);
  const float* gate = tab + mod_offset(s, l, st == ST_O ? 0 : 1, 2);
  const float* scn = !has_next ? nullptr : (st == ST_O ? tab + mod_offset(s, l, 1, 0) : tab + mod_offset(s, l + 1, 0, 0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qd = warp & 3, row = qd * 32 + lane;  // TMEM lane = weight row
  const int Mp = (a.M + 3) & ~3;                   // tokens exchanged per row
  const uint32_t rx = smem_u32(c.work) + kFRx;     // [C][R][Mp] fp32
  const float* rxf = reinterpret_cast<const float*>(c.work + kFRx);
  const uint32_t xbytes = (uint32_t)((C - 1) * R * Mp * 4);
  const int per8 = R / 8, nitems = a.M * per8;
  const int npass = (nitems + kFCompute - 1) / kFCompute;
  // this thread's partial row: own rows straight into this rank's slice of
  // the receive area, the others staged by owner for one bulk copy per peer
  const int owner = row / R, orow = row - owner * R;
  const uint32_t stg = smem_u32(c.work) + kFStg;  // [C][R][Mp] fp32
  const uint32_t slice = (uint32_t)(R * Mp * 4);
  const uint32_t dst = owner == rank ? rx + (uint32_t)rank * slice + (uint32_t)(orow * Mp * 4)
                                     : stg + (uint32_t)owner * slice + (uint32_t)(orow * Mp * 4);
  for (int j = 0; j < nt; ++j) {
    const int t = first + j * a.NC;
    // a. the receive area is free: previous exchange reduced, operand below it
    xchg_open(c, xbytes);
    xopen = true;
    const int slot = it & 1;
    if (!cwait(c, &c.acc_full[slot], (uint32_t)(it >> 1) & 1u)) return false;
    ++it;
    tc_fence_after();
    if (j == 0) FTRACE(c, tr, tb + 2);
    // b. epilogue inputs of the first pass, in flight during the exchange
    EpiIn in;
    auto load_in = [&](int pass) {
      const int idx = c.ct + pass * kFCompute;
      if (idx >= nitems) return;
      const int m = idx / per8, f0 = 128 * t + rank * R + (idx - m * per8) * 8;
      const float* hp = a.h + (size_t)m * s.D + f0;
      f4_to(in.h, ldcg_f4(hp), ldcg_f4(hp + 4));
      f4_to(in.b, ldg_f4(gate + f0), ldg_f4(gate + f0 + 4));
      if (has_next) f4_to(in.sc, ldg_f4(scn + f0), ldg_f4(scn + f0 + 4));
    };
    load_in(0);
    // c. every peer's receive area is free (and so every copy this CTA sent
    //    in the previous exchange has landed: the staging area is free too)
    if (!xchg_ready(c, xn)) return false;
    if (j == 0) FTRACE(c, tr, tb + 3);
    const uint32_t taddr = c.tmem + ((uint32_t)(qd * 32) << 16) + 64u * (uint32_t)slot;
    for (int c0 = 0; c0 < Mp; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + (uint32_t)c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = c0 + 4 * e;
        if (col < Mp) st_shared_f4(dst + (uint32_t)col * 4u, make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]));
      }
    }
    fence_proxy_async_smem();  // the bulk copies read what the threads stored
    tc_fence_before();
    csync();
    if (c.ct == 0) mbar_arrive(&c.acc_empty[slot]);
    if (c.ct < C && c.ct != rank)  // thread q sends the rows rank q owns
      bulk_push(map_cluster(rx + (uint32_t)rank * slice, (uint32_t)c.ct), stg + (uint32_t)c.ct * slice, slice,
                map_cluster(smem_u32(c.rx), (uint32_t)c.ct));
    if (j == 0) FTRACE(c, tr, tb + 4);
    // d. every peer's slice landed
    if (!xchg_wait(c, xn)) return false;
    ++xn;
    xopen = false;
    if (j == 0) FTRACE(c, tr, tb + 5);
    // e. sum the C slices in rank order, then the epilogue of 8 rows
#pragma unroll 1
    for (int pass = 0; pass < npass; ++pass) {  // uniform
      if (pass > 0) load_in(pass);
      const int idx = c.ct + pass * kFCompute;
      const bool valid = idx < nitems;
      const int m = valid ? idx / per8 : 0, j8 = valid ? idx - (idx / per8) * per8 : 0;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      if (valid) {
        const float* p = rxf + (size_t)(j8 * 8) * Mp + m;
        for (int q = 0; q < C; ++q) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += p[(size_t)(q * R + i) * Mp];
        }
      }
      const int f0 = 128 * t + rank * R + j8 * 8;
      float sq = 0.f;
      if (valid) sq = epi_resid(c, m, f0, acc, in, has_next, st == ST_O ? a.yg : a.yq);
      // the per8 threads of one token are adjacent lanes: fixed shuffle tree
      for (int o = 1; o < per8; o <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (valid && j8 == 0 && has_next) (st == ST_O ? a.ss_g : a.ss_q)[(size_t)(t * C + rank) * 64 + m] = sq;
    }
    csync();  // the receive area has been read
  }
  // publish every tile of the stage (one fence)
  __threadfence();
  csync();
  if (c.ct == 0) {
    for (int j = 0; j < nt; ++j) {
      const int t = first + j * a.NC;
      red_release_u32(st == ST_O ? c_ho(a, t) : c_y(a, t), 1u);
    }
  }
  FTRACE(c, tr, tb + 6);
  return true;
}

// Attention on the clusters that hold an attention unit: rank r takes keys
// [r kps, r kps + kps) of the slot in 64-key chunks (online softmax in the
// log2 domain, thread = query row = TMEM lane).  Then every rank stores its
// unnormalised output rows with their running (max, sum) into the rows'
// owner (rank row / R), which weights rank p's rows by exp2(m_p - M) / L
// (M, L over all ranks) and adds them in rank order.  `ac` counts this CTA's
// chunks (barrier phases).
__device__ bool att_stage(const FC& c, int l, int u, int& ac, int& xn, bool& xopen, int& kv_issued) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const AttU au = att_unit(s, a, c.cl, c.rank);
  if (!au.has) return true;
  const int d = s.d, nbox = d / 64, GH = s.G * s.H, C = a.C;
  const uint32_t qbytes = 128u * d * 2u, kvbytes = (uint32_t)CKF * d * 2u;
  const bool tr = u == 1;
  (void)tr;
  FTRACE(c, tr, 40);
  const int slot_row0 = ((l * s.Bmax + au.b) * s.Hkv + au.g) * s.Ptot;
  bool ok = true;
  if (c.ct == 0) {
    ok = wait_ctr(c, c_qkv(a), (unsigned)(a.q_units * (u + 1)));
    if (ok && au.nch > 0) {
      fence_proxy_async_global_f();
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(c.kv_full, qbytes + 2u * kvbytes);
      const int qrow0 = au.bg * GH + au.qt * 128;
      for (int x = 0; x < nbox; ++x) tma_load_2d(c.work + (size_t)x * 128 * 128, c.mp.q, x * 64, qrow0, c.kv_full);
      for (int x = 0; x < nbox; ++x) {
        tma_load_2d(c.work + qbytes + (size_t)x * CKF * 128, c.mp.k, x * 64, slot_row0 + au.start, c.kv_full);
        tma_load_2d(c.work + qbytes + kvbytes + (size_t)x * CKF * 128, c.mp.v, x * 64, slot_row0 + au.start,
                    c.kv_full);
      }
      ++kv_issued;
    }
  }
  FTRACE(c, tr, 41);
  if (!cand(ok)) return false;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qd = warp & 3, r = qd * 32 + lane;
  const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
  const float scale_log2 = rsqrtf((float)d) * 1.4426950408889634f;
  float m_run = -INFINITY, l_run = 0.f;
  for (int ch = 0; ch < au.nch; ++ch) {
    const int acn = ac + ch;
    if (!cwait(c, c.s_full, acn & 1)) return false;
    if (ch == 0) FTRACE(c, tr, 42);
    tc_fence_after();
    float sv[CKF];
#pragma unroll
    for (int j = 0; j < CKF; j += 16) tmem_ld16(c.tmem + lane_off + kColS + j, sv + j);
    tmem_ld_wait();
    const int vc = min(CKF, au.end - (au.start + ch * CKF));
    float cmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < CKF; ++j) {
      sv[j] = j < vc ? sv[j] * scale_log2 : -INFINITY;
      cmax = fmaxf(cmax, sv[j]);
    }
    // lazy rescaling: the reference max moves only when the row max grows by > 8
    const float mx = cmax > m_run + 8.f ? cmax : m_run;
    const float alpha = exp2f(m_run - mx);
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < CKF; ++j) {
      sv[j] = exp2f(sv[j] - mx);
      psum += sv[j];
    }
    l_run = l_run * alpha + psum;
    m_run = mx;
    // S of this chunk completing implies the previous chunk's PV completed
    // (one MMA thread, in order): O may be rescaled and P overwritten
    if (ch > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
      for (int j = 0; j < d; j += 16) {
        float ov[16];
        tmem_ld16(c.tmem + lane_off + kColO + j, ov);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 16; ++t) ov[t] *= alpha;
        tmem_st16(c.tmem + lane_off + kColO + j, ov);
      }
      tmem_st_wait();
    }
    {
      float pk[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) pk[q] = __uint_as_float(pack_bf2(sv[2 * q], sv[2 * q + 1]));
      tmem_st16(c.tmem + lane_off + kColS, pk);
      tmem_st16(c.tmem + lane_off + kColS + 16, pk + 16);
      tmem_st_wait();
    }
    if (vc < CKF) {
      // masked keys have P = 0, but 0 * (NaN or Inf) in V would still poison O
      if (!cwait(c, c.kv_full, acn & 1)) return false;
      uint8_t* vbase = c.work + qbytes + kvbytes;
      const int rows = CKF - vc;
      for (int i = c.ct; i < rows * nbox * 8; i += kFCompute) {
        const int kr = vc + i / (nbox * 8), rem = i % (nbox * 8), x = rem / 8, q = rem % 8;
        *reinterpret_cast<uint4*>(vbase + (size_t)x * CKF * 128 + kr * 128 + q * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    csync();
    if (c.ct == 0) mbar_arrive(c.p_full);
    if (ch + 1 < au.nch) {
      // the next chunk's K and V overwrite this chunk's: wait for its PV
      if (!cwait(c, c.o_full, acn & 1)) return false;
      if (c.ct == 0) {
        mbar_arrive_expect_tx(c.kv_full, 2u * kvbytes);
        const int krow = slot_row0 + au.start + (ch + 1) * CKF;
        for (int x = 0; x < nbox; ++x) {
          tma_load_2d(c.work + qbytes + (size_t)x * CKF * 128, c.mp.k, x * 64, krow, c.kv_full);
          tma_load_2d(c.work + qbytes + kvbytes + (size_t)x * CKF * 128, c.mp.v, x * 64, krow, c.kv_full);
        }
        ++kv_issued;
      }
    }
  }
  ac += au.nch;
  if (au.nch > 0 && !cwait(c, c.o_full, (ac - 1) & 1)) return false;
  tc_fence_after();
  FTRACE(c, tr, 43);

  // -------------------------------------------------- merge in the cluster
  // Rows travel as bf16 (unnormalised partial outputs; the weights are
  // applied in fp32 by the owner): receive area [C][R][d] at the start of
  // the work area, rows staged by owner [C][R][d] at kFAStg, one bulk copy
  // per peer; (max, sum) per row as fp32 stores into the owner's s_st.
  // The work area (q, K, V) is free once every thread is past its last use.
  csync();
  const int R = 128 / C, owner = r / R, orow = r - owner * R;
  const uint32_t slice = (uint32_t)(R * d * 2);
  xchg_open(c, (uint32_t)(C - 1) * (slice + (uint32_t)(R * 8)));
  xopen = true;
  if (!xchg_ready(c, xn)) return false;
  FTRACE(c, tr, 44);
  {
    const bool local = owner == c.rank;
    const uint32_t rx = smem_u32(c.work), stg = smem_u32(c.work) + kFAStg;
    const uint32_t dr = (local ? rx + (uint32_t)c.rank * slice : stg + (uint32_t)owner * slice) + (uint32_t)(orow * d * 2);
    const uint32_t sa = smem_u32(c.s_st) + (uint32_t)((c.rank * R + orow) * 8);
    const float mv = au.nch > 0 ? m_run : -INFINITY, lv = au.nch > 0 ? l_run : 0.f;
    if (local) {
      st_shared_f32(sa, mv);
      st_shared_f32(sa + 4, lv);
    } else {
      st_async_f2(map_cluster(sa, (uint32_t)owner), mv, lv, map_cluster(smem_u32(c.rx), (uint32_t)owner));
    }
    for (int j = 0; j < d; j += 16) {
      float ov[16];
      if (au.nch > 0) {  // uniform over the CTA
        tmem_ld16(c.tmem + lane_off + kColO + j, ov);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) ov[t] = 0.f;
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dr + (uint32_t)j * 2u), "r"(pack_bf2(ov[0], ov[1])),
                   "r"(pack_bf2(ov[2], ov[3])), "r"(pack_bf2(ov[4], ov[5])), "r"(pack_bf2(ov[6], ov[7]))
                   : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dr + (uint32_t)j * 2u + 16u),
                   "r"(pack_bf2(ov[8], ov[9])), "r"(pack_bf2(ov[10], ov[11])), "r"(pack_bf2(ov[12], ov[13])),
                   "r"(pack_bf2(ov[14], ov[15]))
                   : "memory");
    }
    fence_proxy_async_smem();  // the bulk copies read what the threads stored
    tc_fence_before();
    csync();
    if (c.ct < C && c.ct != c.rank)  // thread q sends the rows rank q owns
      bulk_push(map_cluster(rx + (uint32_t)c.rank * slice, (uint32_t)c.ct), stg + (uint32_t)c.ct * slice, slice,
                map_cluster(smem_u32(c.rx), (uint32_t)c.ct));
  }
  if (!xchg_wait(c, xn)) return false;
  ++xn;
  xopen = false;
  FTRACE(c, tr, 45);
  // weight of rank q's slice of row rr: exp2(m_q - M) / L, in s_tmp[rr][q] (R C = 128 floats)
  if (c.ct < R) {
    float mq[16], lq[16];
    float Mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (q < C) {
        mq[q] = c.s_st[(q * R + c.ct) * 2];
        lq[q] = c.s_st[(q * R + c.ct) * 2 + 1];
        Mx = fmaxf(Mx, mq[q]);
      }
    float Ls = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (q < C && lq[q] > 0.f) Ls = fmaf(exp2f(mq[q] - Mx), lq[q], Ls);
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (q < C) c.s_tmp[c.ct * C + q] = (lq[q] > 0.f && Ls > 0.f) ? exp2f(mq[q] - Mx) / Ls : 0.f;
  }
  csync();
  const int per_row = d / 4;
  for (int el = c.ct; el < R * per_row; el += kFCompute) {
    const int rr = el / per_row, c4 = el - rr * per_row;
    const int rq = au.qt * 128 + c.rank * R + rr;
    if (rq >= GH) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < C; ++q) {
      const float w = c.s_tmp[rr * C + q];
      const uint2 p = *reinterpret_cast<const uint2*>(c.work + ((size_t)(q * R + rr) * d + 4 * c4) * 2);
      acc.x = fmaf(w, __uint_as_float(p.x << 16), acc.x);
      acc.y = fmaf(w, __uint_as_float(p.x & 0xFFFF0000u), acc.y);
      acc.z = fmaf(w, __uint_as_float(p.y << 16), acc.z);
      acc.w = fmaf(w, __uint_as_float(p.y & 0xFFFF0000u), acc.w);
    }
    const int hl = rq / s.H, ti = rq - hl * s.H;
    bf16* orow = a.o + (size_t)(au.b * s.H + ti) * s.attn_dim + (au.g * s.G + hl) * d;
    *reinterpret_cast<uint2*>(orow + 4 * c4) = make_uint2(pack_bf2(acc.x, acc.y), pack_bf2(acc.z, acc.w));
  }
  FTRACE(c, tr, 46);
  publish(c, c_att(a));  // its barrier also ends every thread's reads of the area
  FTRACE(c, tr, 47);
  return true;
}

// Token transition for token m = this CTA: (end of step k_out) final
// adaRMSNorm, out_proj, x += dt v; (start of step k_in) h = x W_in^T + b_in,
// its sum of squares and the first norm's operand bf16(h (1 + scale)).
__device__ bool transition(const FC& c, int k_out, int k_in) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  const int m = c.cta;
  if (m >= a.M) return true;
  const int D = s.D, A = s.A;
  const int tid = c.ct, lane = tid & 31, warp = tid >> 5;
  constexpr int nw = kFCompute / 32;
  float* hs = reinterpret_cast<float*>(c.work);  // [D] (the operand area: this CTA's MMAs are done with it)
  float* xs = hs + D;                            // [A]
  float* xrow = a.x + (size_t)m * A;
  if (k_out >= 0) {
    bool ok = true;
    if (tid < 32) ok = wait_ctrs(c, c_y(a, 0), a.d_tiles, (unsigned)a.C * (unsigned)((k_out - a.k_begin) * s.L + s.L));
    if (!cand(ok)) return false;
    const float* tab = a.tables + (size_t)k_out * s.table_rows;
    const float* sc = tab + final_offset(s, 0);
    const float* sh = tab + final_offset(s, 1);
    const float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * kFCompute) {
      const float4 v = ldcg_f4(hrow + j);
      *reinterpret_cast<float4*>(hs + j) = v;
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = csum(c, ss);
    const float rr = rsqrtf(ss / (float)D + s.eps);
    for (int j = 4 * tid; j < D; j += 4 * kFCompute) {
      float4 v = *reinterpret_cast<const float4*>(hs + j);
      const float4 cc = ldg_f4(sc + j), dd = ldg_f4(sh + j);
      v.x = v.x * rr * (1.f + cc.x) + dd.x;
      v.y = v.y * rr * (1.f + cc.y) + dd.y;
      v.z = v.z * rr * (1.f + cc.z) + dd.z;
      v.w = v.w * rr * (1.f + cc.w) + dd.w;
      *reinterpret_cast<float4*>(hs + j) = v;
    }
    csync();
    // v = y W_out^T + b_out: warp w takes outputs w, w + 4, ...; 8 inputs per lane per 256
    const float dtk = __ldg(a.dt + k_out);
    for (int o = warp; o < A; o += nw) {
      float acc = 0.f;
      const bf16* wr = a.w_out + (size_t)o * D;
      for (int j0 = 8 * lane; j0 < D; j0 += 256) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wr + j0));
        const uint32_t wq[4] = {wv.x, wv.y, wv.z, wv.w};
        const float4 y0 = *reinterpret_cast<const float4*>(hs + j0);
        const float4 y1 = *reinterpret_cast<const float4*>(hs + j0 + 4);
        const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc = fmaf(yv[2 * t], __uint_as_float(wq[t] << 16), acc);
          acc = fmaf(yv[2 * t + 1], __uint_as_float(wq[t] & 0xFFFF0000u), acc);
        }
      }
      const float v = warp_sum(acc);
      if (lane == 0) {
        const float xn = __ldcg(xrow + o) + dtk * (v + bf2f(a.b_out[o]));
        xrow[o] = xn;
        xs[o] = xn;
      }
    }
    csync();
  } else {
    for (int o = tid; o < A; o += kFCompute) xs[o] = __ldcg(xrow + o);
    csync();
  }
  if (k_in >= 0) {
    const float* sc0 = a.tables + (size_t)k_in * s.table_rows + mod_offset(s, 0, 0, 0);
    float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * kFCompute) {
      float acc[4];
      {
        const uint2 bv = __ldg(reinterpret_cast<const uint2*>(a.b_in + j));
        acc[0] = __uint_as_float(bv.x << 16);
        acc[1] = __uint_as_float(bv.x & 0xFFFF0000u);
        acc[2] = __uint_as_float(bv.y << 16);
        acc[3] = __uint_as_float(bv.y & 0xFFFF0000u);
      }
      for (int o = 0; o < A; ++o) {
        const uint2 wv = __ldg(reinterpret_cast<const uint2*>(a.w_inT + (size_t)o * D + j));
        const float xv = xs[o];
        acc[0] = fmaf(xv, __uint_as_float(wv.x << 16), acc[0]);
        acc[1] = fmaf(xv, __uint_as_float(wv.x & 0xFFFF0000u), acc[1]);
        acc[2] = fmaf(xv, __uint_as_float(wv.y << 16), acc[2]);
        acc[3] = fmaf(xv, __uint_as_float(wv.y & 0xFFFF0000u), acc[3]);
      }
      *reinterpret_cast<float4*>(hrow + j) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      const float4 cc = ldg_f4(sc0 + j);
      *reinterpret_cast<uint2*>(a.yq + (size_t)m * D + j) =
          make_uint2(pack_bf2(acc[0] * (1.f + cc.x), acc[1] * (1.f + cc.y)),
                     pack_bf2(acc[2] * (1.f + cc.z), acc[3] * (1.f + cc.w)));
      ss = fmaf(acc[0], acc[0], fmaf(acc[1], acc[1], fmaf(acc[2], acc[2], fmaf(acc[3], acc[3], ss))));
    }
    ss = csum(c, ss);
    if (tid == 0) a.ss_t[m] = ss;
  }
  publish(c, c_tr(a));
  csync();  // the work area is reused by the next stage
  return true;
}

__device__ void compute_loop(const FC& c) {
  const Shape& s = *c.s;
  const FlowArgs& a = *c.a;
  int it = 0, sw = 0, ac = 0, xn = 0, kv_issued = 0;
  int opn[4] = {0, 0, 0, 0};
  bool xopen = false;
  if (c.ct < a.B) c.s_len[c.ct] = __ldg(a.lens + c.ct);  // set before the launch, fixed during it
  csync();
  bool ok = transition(c, -1, a.k_begin);
  for (int k = a.k_begin; ok && k < a.k_end; ++k) {
    for (int l = 0; ok && l < s.L; ++l) {
      const int u = (k - a.k_begin) * s.L + l;
      ok = whole_stage(c, ST_Q, k, l, u, sw, opn) && att_stage(c, l, u, ac, xn, xopen, kv_issued) &&
           split_stage(c, ST_O, k, l, u, it, xn, xopen, opn) && whole_stage(c, ST_G, k, l, u, sw, opn) &&
           split_stage(c, ST_D, k, l, u, it, xn, xopen, opn);
    }
    if (ok) ok = transition(c, k, k + 1 < a.k_end ? k + 1 : -1);
  }
  // after an abort, copies this CTA issued may still be in flight, and peers
  // may still be storing into an exchange it had opened: let them land
  if (c.ct == 0) {
    for (int gi = 0; gi < 4; ++gi)
      if (opn[gi] > 0 && !mbar_wait(&c.op_full[gi], (opn[gi] - 1) & 1, kFDrain)) set_error(a.err, DEV_DRAIN);
    if (kv_issued > 0 && !mbar_wait(c.kv_full, (kv_issued - 1) & 1, kFDrain)) set_error(a.err, DEV_DRAIN);
    if (xopen && a.C > 1) (void)mbar_wait(c.rx, (uint32_t)xn & 1u, kFExitWait);
    // after an abort, bulk copies this CTA sent may not have been awaited by
    // their receivers: give them time to read this CTA's staging area (they
    // take microseconds) before the exit barrier
    if (*c.s_abort && (xn > 0 || xopen)) {
      const unsigned long long t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    }
  }
}

__global__ void __launch_bounds__(kFThreads, 1)
    k_flow(const __grid_constant__ CUtensorMap tmWq, const __grid_constant__ CUtensorMap tmWo,
           const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWd,
           const __grid_constant__ CUtensorMap tmYq, const __grid_constant__ CUtensorMap tmO,
           const __grid_constant__ CUtensorMap tmYg, const __grid_constant__ CUtensorMap tmU,
           const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Shape s,
           const __grid_constant__ FlowArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = smem + kFRing * kFBlk + kFWork;
  uint64_t* bar = reinterpret_cast<uint64_t*>(misc);
  FC c{};
  c.s = &s;
  c.a = &a;
  c.mp.w[0] = &tmWq;
  c.mp.w[1] = &tmWo;
  c.mp.w[2] = &tmWg;
  c.mp.w[3] = &tmWd;
  c.mp.x[0] = &tmYq;
  c.mp.x[1] = &tmO;
  c.mp.x[2] = &tmYg;
  c.mp.x[3] = &tmU;
  c.mp.q = &tmQ;
  c.mp.k = &tmK;
  c.mp.v = &tmV;
  c.ring = smem;
  c.work = smem + kFRing * kFBlk;
  // mbarriers
  c.rfull = bar;                   // [kFRing]
  c.rempty = bar + kFRing;         // [kFRing]
  c.op_full = bar + 2 * kFRing;    // [4]
  c.acc_full = c.op_full + 4;      // [2]
  c.acc_empty = c.acc_full + 2;    // [2]
  c.acc_all = c.acc_empty + 2;
  c.kv_full = c.acc_all + 1;
  c.s_full = c.kv_full + 1;
  c.p_full = c.s_full + 1;
  c.o_full = c.p_full + 1;
  c.rx = c.o_full + 1;
  c.rdy = c.rx + 1;
  c.drain = c.rdy + 1;
  c.raw_full = c.drain + 1;        // [kFRawRing]
  const int nbar = (int)(c.raw_full + kFRawRing - bar);
  c.nring = a.w4 ? kFRing - 1 : kFRing;
  c.raw = smem + (kFRing - 1) * kFBlk;  // int4 mode: the fifth bf16 slot holds the packed ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 256);
  c.s_abort = reinterpret_cast<volatile int*>(misc + 260);
  c.s_flag = reinterpret_cast<volatile int*>(misc + 264);
  c.s_rstd = reinterpret_cast<float*>(misc + 512);   // [64]
  c.s_tmp = reinterpret_cast<float*>(misc + 768);    // [512]
  c.s_st = reinterpret_cast<float*>(misc + 2816);    // [C][R][2] = 1 KB
  c.s_len = reinterpret_cast<int*>(misc + 3840);     // [64]
  c.cta = blockIdx.x;
  c.ncta = gridDim.x;
  c.rank = (int)cluster_rank();
  c.cl = blockIdx.x / a.C;
  c.ct = (int)threadIdx.x - 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nbar; ++i) mbar_init(&bar[i], (&bar[i] == c.rdy && a.C > 1) ? (uint32_t)(a.C - 1) : 1u);
    *c.s_abort = 0;
    *c.s_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < 4; ++i) {
      tma_prefetch_desc(c.mp.w[i]);
      tma_prefetch_desc(c.mp.x[i]);
    }
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kFTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *tmem_slot;
  hw_cluster_sync();  // every rank's mbarriers exist before any remote arrival or store

  if (warp == 0) {
    producer_warp(c);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_loop(c);
    __syncwarp();
  } else {
    compute_loop(c);
  }
  tc_fence_before();
  __syncthreads();
  hw_cluster_sync();  // no CTA leaves while a peer may still write its shared memory
  if (warp == 0) tmem_dealloc(c.tmem, kFTmem);
}

}  // namespace

#ifdef PAE_FLOW_TRACE
extern "C" int pae_flow_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_flow_trace, bytes < sizeof(g_flow_trace) ? bytes : sizeof(g_flow_trace));
}
#endif

size_t flow_smem_bytes() { return kFSmem; }

cudaError_t flow_init() {
  cudaError_t e = cudaFuncSetAttribute(k_flow, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFSmem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_flow, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

static void flow_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int C, int NC, cudaStream_t st) {
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(NC * C);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = kFSmem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
}

int flow_max_clusters(int C) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  flow_config(cfg, attr, C, 1, nullptr);
  cfg.numAttrs = 1;  // occupancy of the cluster shape alone
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_flow, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// A cooperative launch guarantees that all clusters are resident together.
// Where the runtime does not take the cooperative attribute together with a
// cluster shape, the plain cluster launch of the same grid (no more clusters
// than fit at once) is used; every wait is bounded either way.
cudaError_t launch_flow(const Shape& s, const CUtensorMap* maps, const FlowArgs& a, cudaStream_t st) {
  static bool cooperative_ok = true;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  flow_config(cfg, attr, a.C, a.NC, st);
  if (!cooperative_ok) cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_flow, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6],
                                     maps[7], maps[8], maps[9], maps[10], s, a);
  if ((e == cudaErrorInvalidValue || e == cudaErrorNotSupported) && cooperative_ok) {
    cudaGetLastError();
    cooperative_ok = false;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_flow, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], maps[7],
                           maps[8], maps[9], maps[10], s, a);
  }
  return e;
}

}  // namespace pae
