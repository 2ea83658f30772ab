// Persistent denoise loop for small batches (B*H <= 64 action tokens).
//
// One cooperative launch runs every Euler step of a pae_denoise call: the
// token transition (final adaRMSNorm, out_proj, Euler update x += dt v,
// in_proj), then per layer the five phases
//   Q  adaRMSNorm + QKV projection (q to the head-major buffer, k/v into the slot)
//   A  GQA attention over [cached prefix | action keys]
//   O  O projection + gated residual
//   G  adaRMSNorm + gate/up projection + GeGLU
//   D  down projection + gated residual
// with one grid barrier after each.  There is no kernel boundary between the
// phases, so the launch/drain latency of ~90 dependent kernels per step is
// gone, and the weights (which do not depend on the activations) stream ahead
// of the barriers.
//
// Per CTA (one per SM, 320 threads):
//   warp 8, lane 0   weight producer: TMA of [128 rows][64] bf16 weight tiles
//                    (128-byte swizzled) into a 5-stage ring, in this CTA's
//                    schedule order, so it runs ahead across phases and layers
//   warp 9, lane 0   MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 in TMEM)
//   warps 0-7        the rest: the token operand of each projection, built in
//                    shared memory (for Q and G the adaRMSNorm is applied here,
//                    from per-token sums of squares the residual phases leave
//                    behind), accumulator reads from TMEM, the split-K
//                    exchange, the epilogues, attention loads and softmax, and
//                    the grid barriers.
// Projections: an output tile is 128 weight rows x 64 tokens; the K range of a
// tile is split over S CTAs so that all SMs stream weights.  Every CTA writes
// its fp32 partial tile to a global workspace, the S CTAs of a tile (2S for
// the gate/up pair) meet on a counter, and each then sums a fixed slice of the
// rows over the partials in split order and applies the epilogue, so results
// are bitwise reproducible.  Attention: one CTA per (request, KV head, 128
// query rows, key range), partials merged the same way.
//
// Every wait is bounded (%globaltimer).  A wait that runs out sets the error
// word and a launch-wide abort flag that all other waits watch, so every CTA
// unwinds; each CTA drains its own copies and MMAs before freeing TMEM.
#include "epilogue.cuh"
#include "launch.cuh"

namespace pae {

namespace {

constexpr int kThreads = 320;
constexpr int kCompute = 256;
constexpr int kRing = 5;
constexpr uint32_t kStage = 16384;          // [128][64] bf16 weight tile
constexpr uint32_t kWork = 128 * 1024;
constexpr uint32_t kMisc = 4096;
constexpr int CK = 64;                      // keys per attention chunk
constexpr long long kDrainNs = 4000000000LL;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 384;           // projection accumulator [384, 448)
constexpr uint32_t kSCol = 256;             // attention scores [256, 320); O at [0, d)
constexpr size_t kPartFloats = 128 * 64;    // one projection partial tile [64 tokens][128 rows]

enum : int { PH_Q = 0, PH_O = 1, PH_G = 2, PH_D = 3 };
enum : int { CT_Q = 0, CT_A = 1, CT_O = 2, CT_G = 3, CT_D = 4 };

constexpr uint32_t kSmemTotal = kRing * kStage + kWork + kMisc + 1024;

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// AND over the threads of named barrier `id` (all `n` of them take part).
// Lanes may leave a bounded wait at different times: reconverge the warp
// before the (warp-aligned) barrier instruction.
__device__ __forceinline__ bool named_and(int id, int n, bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cbar() {
  __syncwarp();
  named_bar(1, kCompute);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Loads of data other CTAs wrote during this launch: L2 only (never a stale L1 line).
__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ uint4 ldcg_u4(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  return (uint32_t)__bfloat16_as_ushort(f2bf(a)) | ((uint32_t)__bfloat16_as_ushort(f2bf(b)) << 16);
}
__device__ __forceinline__ void store4_bf16(bf16* p, float a, float b, float c, float d) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack2(a, b), pack2(c, d));
}
// 8 consecutive bf16 weights as floats (one 16-byte load).
__device__ __forceinline__ void load8w(const bf16* p, float* w) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[2 * i] = __uint_as_float(q[i] << 16);
    w[2 * i + 1] = __uint_as_float(q[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load4w(const bf16* p, float* w) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  w[0] = __uint_as_float(u.x << 16);
  w[1] = __uint_as_float(u.x & 0xFFFF0000u);
  w[2] = __uint_as_float(u.y << 16);
  w[3] = __uint_as_float(u.y & 0xFFFF0000u);
}

// Bounded mbarrier wait that also gives up as soon as this CTA is aborting.
__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity, long long limit_ns,
                                      const volatile int* abort_cta) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_cta) return false;
    if ((long long)(globaltimer_ns() - t0) > limit_ns) return false;
  }
}

struct Bars {
  uint64_t* full;   // [kRing] weight stage landed
  uint64_t* empty;  // [kRing] weight stage consumed by the MMAs
  uint64_t* b_ready;
  uint64_t* acc_full;
  uint64_t* kv_full;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_full;
  uint64_t* drain;
};

struct Maps {
  const CUtensorMap* w[4];
  const CUtensorMap* q;
  const CUtensorMap* k;
  const CUtensorMap* v;
};

struct Ctx {
  const Shape* s;
  const PersistArgs* a;
  Maps maps;
  uint8_t* ring;
  uint8_t* work;
  Bars bars;
  float* s_rstd;  // [64]
  float* s_tmp;   // [256]
  float* s_ml;    // [128][2]
  volatile int* s_abort;
  volatile int* s_ok;
  int* s_loads;  // attention load batches issued (kv_full phases), by compute thread 0
  uint32_t tmem;
  int cta, tid;
};

// Launch-wide abort: record the error, stop this CTA's roles, tell all CTAs.
__device__ void raise_abort(const Ctx& c) {
  *c.s_abort = 1;
  atomicExch(reinterpret_cast<int*>(c.a->ctr + kPersistAbortIdx), 1);
  set_error(c.a->err, DEV_TIMEOUT);
}

// ------------------------------------------------------------ schedule
struct Item {
  bool has;
  int idx, t, sp, kb0, kb1;
};
__device__ __forceinline__ Item gemm_item(const PersistPhase& P, int cta) {
  Item it{};
  it.has = cta < P.nt * P.s;
  if (!it.has) return it;
  it.idx = cta;
  it.t = cta / P.s;
  it.sp = cta - it.t * P.s;
  it.kb0 = it.sp * P.nkb / P.s;
  it.kb1 = (it.sp + 1) * P.nkb / P.s;
  return it;
}

struct AttItem {
  bool has;
  int idx, grp, split, qt, bg, b, g, start, end, nch;
};
__device__ __forceinline__ AttItem att_item(const Shape& s, const PersistArgs& a, int cta) {
  AttItem it{};
  it.has = cta < a.a_items;
  if (!it.has) return it;
  it.idx = cta;
  it.grp = cta / a.a_splits;
  it.split = cta - it.grp * a.a_splits;
  it.qt = it.grp % a.a_qtiles;
  it.bg = it.grp / a.a_qtiles;
  it.b = it.bg / s.Hkv;
  it.g = it.bg - it.b * s.Hkv;
  const int n_valid = __ldg(a.lens + it.b) + s.H;  // slot lengths are fixed during the launch
  it.start = it.split * a.a_kps;
  it.end = min(n_valid, it.start + a.a_kps);
  it.nch = it.end > it.start ? (it.end - it.start + CK - 1) / CK : 0;
  return it;
}

// Attention operands in the work area: Q [128][d], K and V chunks [64][d]
// (as d/64 swizzled boxes), P [128][64] bf16 (over K once S is computed,
// when the K chunk is at least 16 KB).
struct AttLayout {
  uint32_t q, k, v, p;
};
__device__ __forceinline__ AttLayout att_layout(int d) {
  AttLayout L;
  const uint32_t qb = 128u * d * 2u, kvb = (uint32_t)CK * d * 2u;
  L.q = 0;
  L.k = qb;
  L.v = qb + kvb;
  L.p = d >= 128 ? L.k : qb + 2 * kvb;
  return L;
}
__device__ __forceinline__ size_t att_part_stride(int d) { return (size_t)128 * d + 256; }

// ------------------------------------------------------------ compute side
// Rendezvous of the compute threads of several CTAs on a counter; every caller
// has finished its global writes.  Returns false when the launch is aborting.
__device__ bool meet(const Ctx& c, unsigned* ctr, unsigned target) {
  cbar();
  if (c.tid == 0) {
    bool ok = *c.s_abort == 0;
    if (ok) {
      __threadfence();
      red_release_add(ctr, 1u);
      const volatile unsigned* abort_g = c.a->ctr + kPersistAbortIdx;
      if (ld_acquire(ctr) < target) {
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire(ctr) < target) {
          if (*abort_g) {
            ok = false;
            *c.s_abort = 1;
            break;
          }
          if ((long long)(globaltimer_ns() - t0) > c.a->err.wait_ns) {
            ok = false;
            raise_abort(c);
            break;
          }
        }
      }
      __threadfence();
    }
    *c.s_ok = ok ? 1 : 0;
  }
  cbar();
  return *c.s_ok != 0;
}

// Deterministic sum over the 256 compute threads (fixed tree).
__device__ float csum(const Ctx& c, float v) {
  v = warp_sum(v);
  const int lane = c.tid & 31, warp = c.tid >> 5;
  cbar();
  if (lane == 0) c.s_tmp[warp] = v;
  cbar();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kCompute / 32; ++w) t += c.s_tmp[w];
  return t;
}

// rstd[m] = 1 / sqrt(sum over the sum-of-squares slots / D + eps).
__device__ void compute_rstd(const Ctx& c, int nslots) {
  const int r = c.tid & 63, j = c.tid >> 6;
  float acc = 0.f;
#pragma unroll 4
  for (int sl = j; sl < nslots; sl += 4) acc += __ldcg(c.a->ss + (size_t)sl * 64 + r);
  cbar();
  c.s_tmp[j * 64 + r] = acc;
  cbar();
  if (c.tid < 64) {
    const float tot = ((c.s_tmp[r] + c.s_tmp[64 + r]) + c.s_tmp[128 + r]) + c.s_tmp[192 + r];
    c.s_rstd[r] = rsqrtf(tot / (float)c.s->D + c.s->eps);
  }
  cbar();
}

// Token operand of a projection: K blocks kb0..kb1-1 as [64 tokens][64] bf16,
// 128-byte swizzled (16-byte chunk q of row r at position q ^ (r % 8)); rows
// past the last token are zero.  Norm mode: y = h * rstd * (1 + scale) + shift.
__device__ void build_norm(const Ctx& c, int kb0, int kb1, const float* scale, const float* shift) {
  const int n = (kb1 - kb0) * 512;
  const uint32_t wbase = smem_u32(c.work);
  const int M = c.a->M, D = c.s->D;
  const float* h = c.a->h;
#pragma unroll 2
  for (int i = c.tid; i < n; i += kCompute) {
    const int kbl = i >> 9, r = (i >> 3) & 63, q = i & 7;
    const int k = (kb0 + kbl) * 64 + q * 8;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (r < M) {
      const float* hp = h + (size_t)r * D + k;
      const float4 h0 = ldcg4(hp), h1 = ldcg4(hp + 4);
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(scale + k));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(scale + k + 4));
      const float4 t0 = __ldg(reinterpret_cast<const float4*>(shift + k));
      const float4 t1 = __ldg(reinterpret_cast<const float4*>(shift + k + 4));
      const float rs = c.s_rstd[r];
      out.x = pack2(h0.x * rs * (1.f + s0.x) + t0.x, h0.y * rs * (1.f + s0.y) + t0.y);
      out.y = pack2(h0.z * rs * (1.f + s0.z) + t0.z, h0.w * rs * (1.f + s0.w) + t0.w);
      out.z = pack2(h1.x * rs * (1.f + s1.x) + t1.x, h1.y * rs * (1.f + s1.y) + t1.y);
      out.w = pack2(h1.z * rs * (1.f + s1.z) + t1.z, h1.w * rs * (1.f + s1.w) + t1.w);
    }
    st_shared_v4(wbase + kbl * 8192 + r * 128 + ((q ^ (r & 7)) << 4), out);
  }
}
// Copy mode: rows of a bf16 activation matrix [tokens][ld].
__device__ void build_copy(const Ctx& c, int kb0, int kb1, const bf16* src, int ld) {
  const int n = (kb1 - kb0) * 512;
  const uint32_t wbase = smem_u32(c.work);
  const int M = c.a->M;
#pragma unroll 4
  for (int i = c.tid; i < n; i += kCompute) {
    const int kbl = i >> 9, r = (i >> 3) & 63, q = i & 7;
    const int k = (kb0 + kbl) * 64 + q * 8;
    const uint4 v = r < M ? ldcg_u4(src + (size_t)r * ld + k) : make_uint4(0, 0, 0, 0);
    st_shared_v4(wbase + kbl * 8192 + r * 128 + ((q ^ (r & 7)) << 4), v);
  }
}

// Token transition for token m = this CTA: (end of step k_out) final norm,
// out_proj, x += dt v; (start of step k_in) h = x W_in^T + b_in and its sum of
// squares into slot 0.  k_out / k_in < 0: that half is skipped.
__device__ void transition(const Ctx& c, int k_out, int k_in) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  const int m = c.cta;
  if (m >= a.M) return;
  const int D = s.D, A = s.A;
  const int tid = c.tid, lane = tid & 31, warp = tid >> 5;
  constexpr int nw = kCompute / 32;
  float* hs = reinterpret_cast<float*>(c.work);  // [D]
  float* xs = hs + D;                            // [A]
  float* xrow = a.x + (size_t)m * A;
  if (k_out >= 0) {
    const float* tab = a.tables + (size_t)k_out * s.table_rows;
    const float* sc = tab + final_offset(s, 0);
    const float* sh = tab + final_offset(s, 1);
    const float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * kCompute) {
      const float4 v = ldcg4(hrow + j);
      *reinterpret_cast<float4*>(hs + j) = v;
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = csum(c, ss);
    const float r = rsqrtf(ss / (float)D + s.eps);
    for (int j = 4 * tid; j < D; j += 4 * kCompute) {
      float4 v = *reinterpret_cast<const float4*>(hs + j);
      const float4 cc = __ldg(reinterpret_cast<const float4*>(sc + j));
      const float4 dd = __ldg(reinterpret_cast<const float4*>(sh + j));
      v.x = v.x * r * (1.f + cc.x) + dd.x;
      v.y = v.y * r * (1.f + cc.y) + dd.y;
      v.z = v.z * r * (1.f + cc.z) + dd.z;
      v.w = v.w * r * (1.f + cc.w) + dd.w;
      *reinterpret_cast<float4*>(hs + j) = v;
    }
    cbar();
    // v = y W_out^T + b_out: warp w takes outputs w, w + 8, ...; 8 inputs per lane per 256
    const float dtk = __ldg(a.dt + k_out);
    for (int o0 = warp; o0 < A; o0 += 4 * nw) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int j0 = 8 * lane; j0 < D; j0 += 256) {
        float w[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (o0 + u * nw < A) load8w(a.w_out + (size_t)(o0 + u * nw) * D + j0, w[u]);
        const float4 y0 = *reinterpret_cast<const float4*>(hs + j0);
        const float4 y1 = *reinterpret_cast<const float4*>(hs + j0 + 4);
        const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (o0 + u * nw < A)
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[u] = fmaf(yv[t], w[u][t], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int o = o0 + u * nw;
        const float v = warp_sum(acc[u]);
        if (lane == 0 && o < A) {
          const float xn = __ldcg(xrow + o) + dtk * (v + bf2f(a.b_out[o]));
          xrow[o] = xn;
          xs[o] = xn;
        }
      }
    }
    cbar();
  } else {
    for (int o = tid; o < A; o += kCompute) xs[o] = __ldcg(xrow + o);
    cbar();
  }
  if (k_in >= 0) {
    float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * kCompute) {
      float acc[4];
      load4w(a.b_in + j, acc);
      for (int o0 = 0; o0 < A; o0 += 16) {
        float w[16][4];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (o0 + u < A) load4w(a.w_inT + (size_t)(o0 + u) * D + j, w[u]);
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (o0 + u < A) {
            const float xv = xs[o0 + u];
#pragma unroll
            for (int t = 0; t < 4; ++t) acc[t] = fmaf(xv, w[u][t], acc[t]);
          }
      }
      *reinterpret_cast<float4*>(hrow + j) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      ss = fmaf(acc[0], acc[0], fmaf(acc[1], acc[1], fmaf(acc[2], acc[2], fmaf(acc[3], acc[3], ss))));
    }
    ss = csum(c, ss);
    if (tid == 0) a.ss[m] = ss;  // slot 0
  }
  cbar();  // the work area is reused by the next phase
}

// Compute side of one projection phase.  gi counts this CTA's projection
// items (accumulator barrier phases).  Returns false on abort.
__device__ bool gemm_phase(const Ctx& c, int ph, int k, int l, int use, int& gi, int nslots_in) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  const PersistPhase& P = a.ph[ph];
  const Item it = gemm_item(P, c.cta);
  if (!it.has) return true;
  const float* tk = a.tables + (size_t)k * s.table_rows;

  // 1. token operand into the work area, then hand it to the MMA thread
  if (ph == PH_Q || ph == PH_G) {
    compute_rstd(c, nslots_in);
    const int norm = ph == PH_Q ? 0 : 1;
    build_norm(c, it.kb0, it.kb1, tk + mod_offset(s, l, norm, 0), tk + mod_offset(s, l, norm, 1));
  } else if (ph == PH_O) {
    build_copy(c, it.kb0, it.kb1, a.o, s.attn_dim);
  } else {
    build_copy(c, it.kb0, it.kb1, a.u, s.F);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  cbar();
  if (c.tid == 0) mbar_arrive(c.bars.b_ready);

  // 2. accumulator -> fp32 partial [token][row] in the workspace
  const bool w = mwait(c.bars.acc_full, gi & 1, a.err.wait_ns, c.s_abort);
  ++gi;
  if (!named_and(1, kCompute, w)) {
    if (c.tid == 0) raise_abort(c);
    return false;
  }
  tc_fence_after();
  const int warp = c.tid >> 5, lane = c.tid & 31;
  {
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t taddr = c.tmem + ((uint32_t)(quarter * 32) << 16) + kAccCol + half * 32;
    float v0[16], v1[16];
    tmem_ld16(taddr, v0);
    tmem_ld16(taddr + 16, v1);
    tmem_ld_wait();
    float* pt = a.part + (size_t)it.idx * kPartFloats + row;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int m0 = half * 32 + i, m1 = m0 + 16;
      if (m0 < a.M) pt[m0 * 128] = v0[i];
      if (m1 < a.M) pt[m1 * 128] = v1[i];
    }
  }
  tc_fence_before();

  // 3. meet the other CTAs of the reduction group
  const int na = P.na, S = P.s;
  const int g = it.t / na;
  const int ct = ph == PH_Q ? CT_Q : ph == PH_O ? CT_O : ph == PH_G ? CT_G : CT_D;
  if (!meet(c, a.ctr + 1 + ct * kPersistGroups + g, (unsigned)((use + 1) * na * S))) return false;

  // 4. this CTA's row slice, summed over the partials in split order, + epilogue
  const int rr = (it.t - g * na) * S + it.sp;  // reducer index within the group
  const int r0 = rr * P.rp;
  const int r1 = min(128, r0 + P.rp);
  const int n4 = r1 > r0 ? (r1 - r0) / 4 : 0;
  const int M = a.M;
  if (ph == PH_O || ph == PH_D) {
    // Residual phases: n4 is a power of two <= 32, so the n4 units of one
    // token sit in adjacent lanes and its sum of squares is a shuffle tree.
    const float* gate = tk + mod_offset(s, l, ph == PH_O ? 0 : 1, 2);
    const int nu = M * n4;
    const int passes = (64 * 32) / kCompute;
    for (int ps = 0; ps < passes; ++ps) {
      const int u = c.tid + ps * kCompute;
      float sq = 0.f;
      int m = 0, q4 = 0;
      if (u < nu) {
        m = u / n4;
        q4 = u - m * n4;
        const int row = r0 + q4 * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float* pp = a.part + (size_t)(it.t * S) * kPartFloats + (size_t)m * 128 + row;
        for (int q = 0; q < S; ++q) {
          const float4 v = ldcg4(pp + (size_t)q * kPartFloats);
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const int f = it.t * 128 + row;
        float* hp = a.h + (size_t)m * s.D + f;
        float4 hv = ldcg4(hp);
        const float4 gv = __ldg(reinterpret_cast<const float4*>(gate + f));
        hv.x = fmaf(gv.x, acc.x, hv.x);
        hv.y = fmaf(gv.y, acc.y, hv.y);
        hv.z = fmaf(gv.z, acc.z, hv.z);
        hv.w = fmaf(gv.w, acc.w, hv.w);
        *reinterpret_cast<float4*>(hp) = hv;
        sq = fmaf(hv.x, hv.x, fmaf(hv.y, hv.y, fmaf(hv.z, hv.z, hv.w * hv.w)));
      }
      if (n4 > 0) {
        for (int o = 1; o < n4; o <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (u < nu && q4 == 0) a.ss[(size_t)it.idx * 64 + m] = sq;
      }
    }
    if (n4 == 0 && c.tid < 64) a.ss[(size_t)it.idx * 64 + c.tid] = 0.f;
  } else if (ph == PH_Q) {
    const int nu = M * n4;
    const int qd = s.Hq * s.d, kvd = s.Hkv * s.d;
    for (int u = c.tid; u < nu; u += kCompute) {
      const int m = u / n4;
      const int row = r0 + (u - m * n4) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float* pp = a.part + (size_t)(it.t * S) * kPartFloats + (size_t)m * 128 + row;
      for (int q = 0; q < S; ++q) {
        const float4 v = ldcg4(pp + (size_t)q * kPartFloats);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const int f = it.t * 128 + row;
      const int b = m / s.H, ti = m - b * s.H;
      bf16* dst;
      if (f < qd) {
        const int hq = f / s.d, j = f - hq * s.d;
        dst = a.q + ((size_t)(b * s.Hq + hq) * s.H + ti) * s.d + j;
      } else {
        const bool is_v = f >= qd + kvd;
        const int fk = f - qd - (is_v ? kvd : 0);
        const int gg = fk / s.d, j = fk - gg * s.d;
        const size_t off = (((size_t)(l * s.Bmax + b) * s.Hkv + gg) * s.Ptot + __ldg(a.lens + b) + ti) * s.d + j;
        dst = (is_v ? a.vc : a.kc) + off;
      }
      store4_bf16(dst, acc.x, acc.y, acc.z, acc.w);
    }
  } else {  // PH_G: gate tile 2g and up tile 2g+1, S partials each
    const int nu = M * n4;
    for (int u = c.tid; u < nu; u += kCompute) {
      const int m = u / n4;
      const int row = r0 + (u - m * n4) * 4;
      float4 ga = make_float4(0.f, 0.f, 0.f, 0.f), ua = ga;
      const float* pg = a.part + (size_t)(2 * g * S) * kPartFloats + (size_t)m * 128 + row;
      const float* pu = pg + (size_t)S * kPartFloats;
      for (int q = 0; q < S; ++q) {
        const float4 v = ldcg4(pg + (size_t)q * kPartFloats);
        const float4 x = ldcg4(pu + (size_t)q * kPartFloats);
        ga.x += v.x;
        ga.y += v.y;
        ga.z += v.z;
        ga.w += v.w;
        ua.x += x.x;
        ua.y += x.y;
        ua.z += x.z;
        ua.w += x.w;
      }
      const int f = g * 128 + row;
      store4_bf16(a.u + (size_t)m * s.F + f, gelu_tanh_bf16out(ga.x) * ua.x, gelu_tanh_bf16out(ga.y) * ua.y,
                  gelu_tanh_bf16out(ga.z) * ua.z, gelu_tanh_bf16out(ga.w) * ua.w);
    }
  }
  return true;
}

// Issue the TMA loads of chunk `ch` (and Q with the first chunk).
__device__ void att_load(const Ctx& c, const AttItem& it, int l, int ch) {
  const Shape& s = *c.s;
  const int d = s.d, nbox = d / 64;
  const AttLayout L = att_layout(d);
  const uint32_t kvb = (uint32_t)CK * d * 2u;
  const bool with_q = ch == 0;
  ++*c.s_loads;
  mbar_arrive_expect_tx(c.bars.kv_full, 2 * kvb + (with_q ? 128u * d * 2u : 0u));
  if (with_q) {
    const int qrow0 = it.bg * s.G * s.H + it.qt * 128;
    for (int x = 0; x < nbox; ++x) tma_load_2d(c.work + L.q + x * 128 * 128, c.maps.q, x * 64, qrow0, c.bars.kv_full);
  }
  const int krow = ((l * s.Bmax + it.b) * s.Hkv + it.g) * s.Ptot + it.start + ch * CK;
  for (int x = 0; x < nbox; ++x) {
    tma_load_2d(c.work + L.k + x * CK * 128, c.maps.k, x * 64, krow, c.bars.kv_full);
    tma_load_2d(c.work + L.v + x * CK * 128, c.maps.v, x * 64, krow, c.bars.kv_full);
  }
}

// Compute side of the attention phase; `ac` counts this CTA's key chunks
// (barrier phases of kv_full / s_full / p_full / o_full).
__device__ bool att_phase(const Ctx& c, int l, int use, int& ac) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  const AttItem it = att_item(s, a, c.cta);
  if (!it.has) return true;
  const int d = s.d, nbox = d / 64;
  const AttLayout L = att_layout(d);
  const int warp = c.tid >> 5, lane = c.tid & 31;
  const float scale_log2 = rsqrtf((float)d) * 1.4426950408889634f;
  const int GH = s.G * s.H;
  const long long wl = a.err.wait_ns;

  if (c.tid == 0 && it.nch > 0) {
    fence_proxy_async_global();  // q and the action keys were written by generic stores of other CTAs
    att_load(c, it, l, 0);
  }
  bool ok = true;
  if (warp < 4) {
    // -------------------------------------------- softmax: thread = query row
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    for (int ch = 0; ch < it.nch; ++ch) {
      const int acn = ac + ch;
      const bool w1 = mwait(c.bars.s_full, acn & 1, wl, c.s_abort);
      if (!named_and(2, 128, w1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[CK];
#pragma unroll
      for (int j = 0; j < CK; j += 16) tmem_ld16(c.tmem + lane_off + kSCol + j, sv + j);
      tmem_ld_wait();
      const int vc = min(CK, it.end - (it.start + ch * CK));
      float cmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < CK; ++j) {
        sv[j] = j < vc ? sv[j] * scale_log2 : -INFINITY;
        cmax = fmaxf(cmax, sv[j]);
      }
      // lazy rescaling: the reference max moves only when the row max grows by > 8
      const float mx = cmax > m_run + 8.f ? cmax : m_run;
      const float alpha = exp2f(m_run - mx);
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < CK; ++j) {
        sv[j] = exp2f(sv[j] - mx);
        psum += sv[j];
      }
      l_run = l_run * alpha + psum;
      m_run = mx;
      if (ch > 0) {
        // the previous PV is done (O may be rescaled; P and V may be rewritten)
        const bool w2 = mwait(c.bars.o_full, (acn - 1) & 1, wl, c.s_abort);
        if (!named_and(2, 128, w2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha < 1.f)) {
          for (int j = 0; j < d; j += 16) {
            float ov[16];
            tmem_ld16(c.tmem + lane_off + j, ov);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 16; ++t) ov[t] *= alpha;
            tmem_st16(c.tmem + lane_off + j, ov);
          }
          tmem_st_wait();
        }
      }
      const uint32_t p_row = smem_u32(c.work + L.p) + r * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t addr = p_row + (((uint32_t)q ^ (uint32_t)(r & 7)) << 4);
        st_shared_v4(addr, make_uint4(pack2(sv[q * 8 + 0], sv[q * 8 + 1]), pack2(sv[q * 8 + 2], sv[q * 8 + 3]),
                                      pack2(sv[q * 8 + 4], sv[q * 8 + 5]), pack2(sv[q * 8 + 6], sv[q * 8 + 7])));
      }
      bool w3 = true;
      if (vc < CK) {
        // masked keys have P = 0, but 0 * (NaN or Inf) in V would still poison O
        w3 = mwait(c.bars.kv_full, acn & 1, kDrainNs, c.s_abort);
        if (w3) {
          uint8_t* vbase = c.work + L.v;
          const int rows = CK - vc;
          for (int i = r; i < rows * nbox * 8; i += 128) {
            const int kr = vc + i / (nbox * 8), rem = i % (nbox * 8), x = rem / 8, q = rem % 8;
            *reinterpret_cast<uint4*>(vbase + x * CK * 128 + kr * 128 + q * 16) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (!named_and(2, 128, w3)) {
        ok = false;
        break;
      }
      if (warp == 0) {
        if (lane == 0) mbar_arrive(c.bars.p_full);
        if (ch + 1 < it.nch) {
          // the next chunk's K overwrites P and its V the current V: wait for this PV
          const bool w5 = __all_sync(0xffffffffu, mwait(c.bars.o_full, acn & 1, wl, c.s_abort));
          if (lane == 0) {
            if (w5)
              att_load(c, it, l, ch + 1);
            else
              raise_abort(c);
          }
        }
        __syncwarp();
      }
    }
    c.s_ml[2 * r] = ok && it.nch > 0 ? m_run : -INFINITY;
    c.s_ml[2 * r + 1] = ok && it.nch > 0 ? l_run : 0.f;
  }
  ok = named_and(1, kCompute, ok);
  if (ok && it.nch > 0) {
    const bool w4 = mwait(c.bars.o_full, (ac + it.nch - 1) & 1, wl, c.s_abort);
    ok = named_and(1, kCompute, w4);
  }
  ac += it.nch;
  if (!ok) {
    if (c.tid == 0) raise_abort(c);
    return false;
  }
  tc_fence_after();

  // -------------------------------------------- O rows out of TMEM
  // warp w reads rows 32*(w%4).. and columns [w/4 * d/2, +d/2)
  const int Sa = a.a_splits;
  {
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int c0 = half * (d / 2);
    const int rq = it.qt * 128 + row;
    if (Sa == 1) {
      const float lr = c.s_ml[2 * row + 1];
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      const int hl = rq / s.H, ti = rq - hl * s.H;
      bf16* orow = a.o + (size_t)(it.b * s.H + ti) * s.attn_dim + (it.g * s.G + hl) * d;
      for (int j = c0; j < c0 + d / 2; j += 16) {
        float ov[16];
        if (it.nch > 0) {
          tmem_ld16(c.tmem + lane_off + j, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int t = 0; t < 16; ++t) ov[t] = 0.f;
        }
        if (rq < GH) {
          uint4* dst = reinterpret_cast<uint4*>(orow + j);
          dst[0] = make_uint4(pack2(ov[0] * inv, ov[1] * inv), pack2(ov[2] * inv, ov[3] * inv),
                              pack2(ov[4] * inv, ov[5] * inv), pack2(ov[6] * inv, ov[7] * inv));
          dst[1] = make_uint4(pack2(ov[8] * inv, ov[9] * inv), pack2(ov[10] * inv, ov[11] * inv),
                              pack2(ov[12] * inv, ov[13] * inv), pack2(ov[14] * inv, ov[15] * inv));
        }
      }
    } else {
      float* pr = a.part + (size_t)it.idx * att_part_stride(d);
      if (it.nch > 0) {
        for (int j = c0; j < c0 + d / 2; j += 16) {
          float ov[16];
          tmem_ld16(c.tmem + lane_off + j, ov);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(pr + (size_t)row * d + j);
#pragma unroll
          for (int t = 0; t < 4; ++t) dst[t] = make_float4(ov[4 * t], ov[4 * t + 1], ov[4 * t + 2], ov[4 * t + 3]);
        }
      }
      if (half == 0)
        *reinterpret_cast<float2*>(pr + (size_t)128 * d + 2 * row) = make_float2(c.s_ml[2 * row], c.s_ml[2 * row + 1]);
    }
  }
  tc_fence_before();
  if (Sa == 1) return true;

  // -------------------------------------------- split-KV merge
  if (!meet(c, a.ctr + 1 + CT_A * kPersistGroups + it.grp, (unsigned)((use + 1) * Sa))) return false;
  const int rpa = (128 + Sa - 1) / Sa;
  const int rb = it.split * rpa, re = min(128, rb + rpa);
  const int per_row = d / 4;
  const size_t stride = att_part_stride(d);
  const float* base = a.part + (size_t)(it.grp * Sa) * stride;
  for (int el = c.tid; el < (re - rb) * per_row; el += kCompute) {
    const int row = rb + el / per_row, c4 = el - (el / per_row) * per_row;
    const int rq = it.qt * 128 + row;
    if (rq >= GH) continue;
    float Mx = -INFINITY;
    for (int q = 0; q < Sa; ++q) Mx = fmaxf(Mx, __ldcg(base + (size_t)q * stride + (size_t)128 * d + 2 * row));
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, wsum = 0.f;
    for (int q = 0; q < Sa; ++q) {
      const float* pq = base + (size_t)q * stride;
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(pq + (size_t)128 * d + 2 * row));
      if (!(ml.y > 0.f)) continue;
      const float wq = exp2f(ml.x - Mx);
      const float4 v = ldcg4(pq + (size_t)row * d + c4 * 4);
      wsum = fmaf(wq, ml.y, wsum);
      acc0 = fmaf(wq, v.x, acc0);
      acc1 = fmaf(wq, v.y, acc1);
      acc2 = fmaf(wq, v.z, acc2);
      acc3 = fmaf(wq, v.w, acc3);
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const int hl = rq / s.H, ti = rq - hl * s.H;
    bf16* orow = a.o + (size_t)(it.b * s.H + ti) * s.attn_dim + (it.g * s.G + hl) * d;
    store4_bf16(orow + c4 * 4, acc0 * inv, acc1 * inv, acc2 * inv, acc3 * inv);
  }
  return true;
}

__device__ void compute_loop(const Ctx& c) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  int gi = 0, ac = 0;
  unsigned nbar = 0;
  const unsigned ncta = (unsigned)a.ncta;
  unsigned* gctr = a.ctr;
  const int slots_o = a.ph[PH_O].nt * a.ph[PH_O].s;
  const int slots_d = a.ph[PH_D].nt * a.ph[PH_D].s;
  bool ok = true;
  for (int k = a.k_begin; ok && k < a.k_end; ++k) {
    transition(c, k > a.k_begin ? k - 1 : -1, k);
    ok = meet(c, gctr, ++nbar * ncta);
    for (int l = 0; ok && l < s.L; ++l) {
      const int use = (k - a.k_begin) * s.L + l;
      ok = gemm_phase(c, PH_Q, k, l, use, gi, l == 0 ? 1 : slots_d) && meet(c, gctr, ++nbar * ncta);
      ok = ok && att_phase(c, l, use, ac) && meet(c, gctr, ++nbar * ncta);
      ok = ok && gemm_phase(c, PH_O, k, l, use, gi, 0) && meet(c, gctr, ++nbar * ncta);
      ok = ok && gemm_phase(c, PH_G, k, l, use, gi, slots_o) && meet(c, gctr, ++nbar * ncta);
      ok = ok && gemm_phase(c, PH_D, k, l, use, gi, 0) && meet(c, gctr, ++nbar * ncta);
    }
  }
  if (ok) transition(c, a.k_end - 1, -1);
  // after an abort, attention copies may still be in flight: let the last land
  if (c.tid == 0 && *c.s_loads > 0 && !mbar_wait(c.bars.kv_full, (*c.s_loads - 1) & 1, kDrainNs))
    set_error(a.err, DEV_DRAIN);
}

// ------------------------------------------------------------ weight producer
__device__ void producer_loop(const Ctx& c) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  const uint64_t pol = policy_evict_first();  // weights are streamed once per step
  int n = 0;
  bool ok = true;
  for (int k = a.k_begin; ok && k < a.k_end; ++k)
    for (int l = 0; ok && l < s.L; ++l)
      for (int ph = 0; ok && ph < 4; ++ph) {
        const PersistPhase& P = a.ph[ph];
        const Item it = gemm_item(P, c.cta);
        if (!it.has) continue;
        const int row0 = l * P.wrows + it.t * 128;
        for (int kb = it.kb0; kb < it.kb1; ++kb, ++n) {
          const int st = n % kRing;
          if (n >= kRing && !mwait(&c.bars.empty[st], ((n / kRing) & 1) ^ 1, a.err.wait_ns, c.s_abort)) {
            if (!*c.s_abort) raise_abort(c);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&c.bars.full[st], kStage);
          tma_load_2d_hint(c.ring + (size_t)st * kStage, c.maps.w[ph], kb * 64, row0, &c.bars.full[st], pol);
        }
      }
  // copies still in flight must land before the CTA exits
  for (int j = n > kRing ? n - kRing : 0; j < n; ++j)
    if (!mbar_wait(&c.bars.full[j % kRing], (j / kRing) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
}

// ------------------------------------------------------------ MMA issuer
__device__ void mma_loop(const Ctx& c) {
  const Shape& s = *c.s;
  const PersistArgs& a = *c.a;
  const long long wl = a.err.wait_ns;
  const uint32_t idesc_g = idesc_bf16(128, 64);
  const int d = s.d;
  const uint32_t idesc_s = idesc_bf16(128, CK);
  const uint32_t idesc_o = idesc_bf16(128, d, 0, 1);
  const AttLayout L = att_layout(d);
  const uint32_t work = smem_u32(c.work);
  const uint32_t ring = smem_u32(c.ring);
  int n = 0, gi = 0, ac = 0;
  bool ok = true;
  for (int k = a.k_begin; ok && k < a.k_end; ++k)
    for (int l = 0; ok && l < s.L; ++l)
      for (int ph5 = 0; ok && ph5 < 5; ++ph5) {
        if (ph5 == 1) {
          // attention: S = Q K^T, then O (+)= P V per 64-key chunk
          const AttItem it = att_item(s, a, c.cta);
          if (!it.has) continue;
          for (int ch = 0; ch < it.nch; ++ch) {
            const int acn = ac + ch;
            if (!mwait(c.bars.kv_full, acn & 1, wl, c.s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int k16 = 0; k16 < d / 16; ++k16) {
              const int x = k16 >> 2, w = (k16 & 3) * 32;
              const uint64_t ad = sw128_desc(work + L.q + x * 128 * 128 + w, 16, 1024);
              const uint64_t bd = sw128_desc(work + L.k + x * CK * 128 + w, 16, 1024);
              umma_bf16(c.tmem + kSCol, ad, bd, idesc_s, k16 > 0 ? 1u : 0u);
            }
            umma_commit(c.bars.s_full);
            if (!mwait(c.bars.p_full, acn & 1, wl, c.s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int k16 = 0; k16 < CK / 16; ++k16) {
              const uint64_t ad = sw128_desc(work + L.p + k16 * 32, 16, 1024);
              const uint64_t bd = sw128_desc(work + L.v + k16 * 16 * 128, CK * 128, 1024);
              umma_bf16(c.tmem, ad, bd, idesc_o, (ch > 0 || k16 > 0) ? 1u : 0u);
            }
            umma_commit(c.bars.o_full);
          }
          ac += it.nch;
          continue;
        }
        const int ph = ph5 == 0 ? PH_Q : ph5 - 1;
        const Item it = gemm_item(a.ph[ph], c.cta);
        if (!it.has) continue;
        if (!mwait(c.bars.b_ready, gi & 1, wl, c.s_abort)) {
          ok = false;
          break;
        }
        ++gi;
        tc_fence_after();
        for (int kb = it.kb0; kb < it.kb1; ++kb, ++n) {
          const int st = n % kRing;
          if (!mwait(&c.bars.full[st], (n / kRing) & 1, wl, c.s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = ring + (uint32_t)st * kStage;
          const uint32_t sb = work + (uint32_t)(kb - it.kb0) * 8192u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(c.tmem + kAccCol, sw128_desc(sa + kk * 32, 16, 1024), sw128_desc(sb + kk * 32, 16, 1024), idesc_g,
                      (kb > it.kb0 || kk > 0) ? 1u : 0u);
          umma_commit(&c.bars.empty[st]);
        }
        if (!ok) break;
        umma_commit(c.bars.acc_full);
      }
  if (!ok && !*c.s_abort) raise_abort(c);
  // every MMA this thread issued must finish before TMEM is freed
  umma_commit(c.bars.drain);
  if (!mbar_wait(c.bars.drain, 0, kDrainNs)) set_error(a.err, DEV_DRAIN);
}

__global__ void __launch_bounds__(kThreads, 1)
    k_persistent(const __grid_constant__ CUtensorMap tmWq, const __grid_constant__ CUtensorMap tmWo,
                 const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWd,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Shape s,
                 const __grid_constant__ PersistArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = smem + kRing * kStage + kWork;
  uint64_t* bar = reinterpret_cast<uint64_t*>(misc);
  Ctx c{};
  c.s = &s;
  c.a = &a;
  c.maps.w[0] = &tmWq;
  c.maps.w[1] = &tmWo;
  c.maps.w[2] = &tmWg;
  c.maps.w[3] = &tmWd;
  c.maps.q = &tmQ;
  c.maps.k = &tmK;
  c.maps.v = &tmV;
  c.ring = smem;
  c.work = smem + kRing * kStage;
  c.bars.full = bar;
  c.bars.empty = bar + kRing;
  c.bars.b_ready = bar + 2 * kRing;
  c.bars.acc_full = bar + 2 * kRing + 1;
  c.bars.kv_full = bar + 2 * kRing + 2;
  c.bars.s_full = bar + 2 * kRing + 3;
  c.bars.p_full = bar + 2 * kRing + 4;
  c.bars.o_full = bar + 2 * kRing + 5;
  c.bars.drain = bar + 2 * kRing + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 256);
  c.s_abort = reinterpret_cast<volatile int*>(misc + 260);
  c.s_ok = reinterpret_cast<volatile int*>(misc + 264);
  c.s_loads = reinterpret_cast<int*>(misc + 268);
  c.s_rstd = reinterpret_cast<float*>(misc + 512);   // [64]
  c.s_tmp = reinterpret_cast<float*>(misc + 768);    // [256]
  c.s_ml = reinterpret_cast<float*>(misc + 1792);    // [128][2]
  c.cta = blockIdx.x;
  c.tid = threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * kRing + 7; ++i) mbar_init(&bar[i], 1);
    *c.s_abort = 0;
    *c.s_ok = 0;
    *c.s_loads = 0;
    fence_mbar_init();
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(c.maps.w[i]);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) producer_loop(c);
    __syncwarp();
  } else if (warp == 9) {
    if (lane == 0) mma_loop(c);
    __syncwarp();
  } else {
    compute_loop(c);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(c.tmem, kTmemCols);
}

}  // namespace

size_t persist_smem_bytes() { return kSmemTotal; }

cudaError_t persist_init() {
  return cudaFuncSetAttribute(k_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTotal);
}

cudaError_t launch_persistent(const Shape& s, const CUtensorMap* maps, const PersistArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.ncta);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemTotal;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_persistent, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], s, a);
}

}  // namespace pae
