// Weight-streaming projection GEMM on the 5th-generation tensor cores.
//
//   out[m][f] = sum_k X[m][k] W[f][k]   followed by one of the epilogues
//   (q/k/v scatter, gated residual, GeGLU).
//
// The weights are the MMA's M side (128 rows per tile, or 2 x 128 for the
// interleaved gate/up tile) and the action tokens are its N side, so a chunk of
// 50 tokens costs one N=64 MMA per 16-wide K step instead of padding tokens to
// 128.  Per CTA:
//   warp 0 / lane 0  TMA producer: weight tile [128*NA][64] and token tile
//                    [tn][64] per stage, both 128-byte swizzled, into a ring
//   warp 1 / lane 0  MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 in TMEM)
//   warps 0-7        epilogue: tcgen05.ld of the accumulator (thread = weight
//                    row = output feature, 16 token columns per load; the two
//                    warpgroups take alternate 16-token chunks, each warp on
//                    its own with the next chunk's load in flight)
// Split-K: the grid.y CTAs of one output tile form a thread-block cluster;
// each CTA pushes its fp32 partial rows into the owning rank's shared memory
// (distributed shared memory stores), and after one cluster barrier every
// rank sums its 1/S slice of the rows over all sources in rank order (thread =
// 4 rows x 1 token, float4 per source), so results are bitwise reproducible
// and no partial touches global memory.
// The weight loads of the first ring are issued before griddepcontrol.wait, so
// under programmatic dependent launch they overlap the previous kernel.
// int4 weights (W4A16): TMA brings the packed [rows][32 bytes] tile per K
// block; warps 4-7 dequantise it into the bf16 A tile (code * group scale,
// rounded once) and arrive on a barrier the MMA thread waits for; the rest of
// the pipeline and the epilogues are shared with the bf16 path.
// In-kernel adaRMSNorm (small batches): the token operand comes from the fp32
// residual stream h, TMA'd per K block into a staging tile; warps 4-7 turn it
// into y = h * rstd * (1 + scale) + shift (bf16, swizzled) and arrive on the
// same barrier.  rstd comes from per-token sum-of-squares slots that the
// residual projections' split-K epilogue writes (one per tile and rank).
#include "epilogue.cuh"
#include "launch.cuh"

namespace pae {

namespace {

// Loads and MMAs always finish in bounded time; waits for them after an abort
// (draining) get this fixed bound instead of the short pipeline limit.
constexpr long long kDrainNs = 4000000000LL;

__host__ __device__ inline uint32_t tmem_cols_for(int n) {
  uint32_t c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

struct TcSmemLayout {
  uint32_t a_bytes, b_bytes, raw_bytes, h_bytes, stage_bytes, recv_off, recv_bytes, bar_off, norm_off, rs_off, total;
};

// Per stage: the bf16 weight tile A ([128*na][64], 128-byte swizzled), the
// token tile B ([tn][64], swizzled) and, for int4 weights, the raw packed tile
// ([128*na][32 bytes]) that the dequantising warps turn into A.  The split-K
// receive buffer ([na][src][token][R] fp32, na*tn*128 floats) follows the ring
// or, when p.recv_alias, overlays it (then an extra cluster barrier makes sure
// every peer's MMAs are done with its ring before anyone pushes).
__host__ __device__ inline TcSmemLayout tc_layout(int na, const TcPlan& p, bool w4, bool norm = false) {
  TcSmemLayout L;
  L.a_bytes = (uint32_t)na * 128u * 128u;
  L.b_bytes = (uint32_t)p.tn * 128u;
  L.raw_bytes = w4 ? (uint32_t)na * 128u * 32u : 0u;
  // norm: fp32 [tn][64] residual staging at the B position; the bf16 B tile is
  // written over its front half once every thread has read its chunks
  L.h_bytes = norm ? (uint32_t)p.tn * 128u : 0u;
  L.stage_bytes = L.a_bytes + L.b_bytes + L.raw_bytes + L.h_bytes;
  const uint32_t ring = L.stage_bytes * (uint32_t)p.stages;
  L.recv_bytes = p.splits > 1 ? (uint32_t)na * (uint32_t)p.tn * 128u * 4u : 0u;
  L.recv_off = p.recv_alias ? 0u : ring;
  const uint32_t used = p.recv_alias ? (ring > L.recv_bytes ? ring : L.recv_bytes) : ring + L.recv_bytes;
  L.bar_off = (used + 15u) & ~15u;
  L.norm_off = L.bar_off + 512;  // (barriers) then rstd [64] + partial sums [2][64]
  L.rs_off = L.norm_off + (norm ? 768u : 0u);  // factored adaRMSNorm: rstd of the tile's tokens [256]
  L.total = L.rs_off + 1024u + 1024u;  // + slack for 1024-byte alignment
  return L;
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void store16_bf16(bf16* p, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = (uint32_t)__bfloat16_as_ushort(f2bf(v[2 * i])) | ((uint32_t)__bfloat16_as_ushort(f2bf(v[2 * i + 1])) << 16);
  uint4* d = reinterpret_cast<uint4*>(p);
  d[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

__device__ __forceinline__ void store8_bf16(bf16* p, const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = (uint32_t)__bfloat16_as_ushort(f2bf(v[2 * i])) | ((uint32_t)__bfloat16_as_ushort(f2bf(v[2 * i + 1])) << 16);
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Where the head `head` of the q/k block (EPI_QKV: q heads then k heads) or of
// the prefix keys (EPI_PREFIX) of token m starts, and that token's position.
template <int EPI>
__device__ __forceinline__ bf16* rot_head_base(const Shape& s, const EpiArgs& e, int m, int head, int len, int& pos) {
  if constexpr (EPI == EPI_PREFIX) {
    pos = m;
    return static_cast<bf16*>(e.kc) + (((size_t)(e.layer * s.Bmax + e.prefix_row) * s.Hkv + head) * s.Ptot + m) * s.d;
  } else {
    const int b = m / s.H, t = m - b * s.H;
    pos = len + t;
    if (head < s.Hq) return static_cast<bf16*>(e.q) + ((size_t)(b * s.Hq + head) * s.H + t) * s.d;
    return static_cast<bf16*>(e.kc) +
           (((size_t)(e.layer * s.Bmax + b) * s.Hkv + (head - s.Hq)) * s.Ptot + len + t) * s.d;
  }
}

// Epilogue of 16 consecutive output features f..f+15 of token m (v holds the
// accumulators; for GeGLU already gelu(gate) * up).  16 divides head_dim and
// 128, so the run never crosses a q/k/v head.  Rotated heads: the 16 stored
// rows are 8 pairs, written to channels i0..i0+7 and i0+d/2..i0+d/2+7.
template <int EPI>
__device__ __forceinline__ void epi_vec16(const Shape& s, const EpiArgs& e, int m, int f, const float* v) {
  if constexpr (EPI == EPI_QKV || EPI == EPI_PREFIX) {
    const int rot_rows = (EPI == EPI_QKV ? s.Hq + s.Hkv : s.Hkv) * s.d;
    if (e.rope_cs && f < rot_rows) {
      const int head = f / s.d, i0 = (f - head * s.d) >> 1;
      int pos;
      const int len = EPI == EPI_QKV ? e.lens[m / s.H] : 0;
      bf16* base = rot_head_base<EPI>(s, e, m, head, len, pos);
      float lo[8], hi[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        lo[u] = v[2 * u];
        hi[u] = v[2 * u + 1];
        rope_turn(e.rope_cs, s.d, pos, i0 + u, lo[u], hi[u]);
      }
      store8_bf16(base + i0, lo);
      store8_bf16(base + i0 + (s.d >> 1), hi);
      return;
    }
  }
  if constexpr (EPI == EPI_PREFIX) {
    const int kvd = s.Hkv * s.d;
    const bool is_v = f >= kvd;
    const int fk = f - (is_v ? kvd : 0);
    const int g = fk / s.d, j = fk - g * s.d;
    const size_t off = (((size_t)(e.layer * s.Bmax + e.prefix_row) * s.Hkv + g) * s.Ptot + m) * s.d + j;
    store16_bf16(static_cast<bf16*>(is_v ? e.vc : e.kc) + off, v);
    return;
  }
  if constexpr (EPI == EPI_RESID) {
    float* hp = e.h + (size_t)m * s.D + f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 h4 = reinterpret_cast<float4*>(hp)[q];
      const float4 g4 = reinterpret_cast<const float4*>(e.gate + f)[q];
      h4.x = fmaf(g4.x, v[4 * q], h4.x);
      h4.y = fmaf(g4.y, v[4 * q + 1], h4.y);
      h4.z = fmaf(g4.z, v[4 * q + 2], h4.z);
      h4.w = fmaf(g4.w, v[4 * q + 3], h4.w);
      reinterpret_cast<float4*>(hp)[q] = h4;
    }
  } else if constexpr (EPI == EPI_GEGLU) {
    store16_bf16(static_cast<bf16*>(e.u) + (size_t)m * s.F + f, v);
  } else {
    const int b = m / s.H, t = m - b * s.H;
    const int qd = s.Hq * s.d;
    if (f < qd) {
      const int hq = f / s.d, j = f - hq * s.d;
      store16_bf16(static_cast<bf16*>(e.q) + ((size_t)(b * s.Hq + hq) * s.H + t) * s.d + j, v);
    } else {
      const int kvd = s.Hkv * s.d;
      const bool is_v = f >= qd + kvd;
      const int fk = f - qd - (is_v ? kvd : 0);
      const int g = fk / s.d, j = fk - g * s.d;
      const size_t off = (((size_t)(e.layer * s.Bmax + b) * s.Hkv + g) * s.Ptot + e.lens[b] + t) * s.d + j;
      store16_bf16(static_cast<bf16*>(is_v ? e.vc : e.kc) + off, v);
    }
  }
}

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ float4 ld_shared_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void add4(float4& a, const float4 b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

__device__ __forceinline__ void store4_bf16(bf16* p, float x, float y, float z, float w) {
  const uint32_t lo = (uint32_t)__bfloat16_as_ushort(f2bf(x)) | ((uint32_t)__bfloat16_as_ushort(f2bf(y)) << 16);
  const uint32_t hi = (uint32_t)__bfloat16_as_ushort(f2bf(z)) | ((uint32_t)__bfloat16_as_ushort(f2bf(w)) << 16);
  *reinterpret_cast<uint2*>(p) = make_uint2(lo, hi);
}

// Epilogue of 4 consecutive output features f..f+3 of token m from the
// reduced accumulators a0 (and a1, the up projection, for GeGLU); h4 is the
// residual stream there and g4 the gate (gated residual), len the slot length
// of the token's request (k / v rows).  4 divides head_dim, so the run never
// crosses a head.
template <int EPI>
__device__ __forceinline__ void epi_vec4(const Shape& s, const EpiArgs& e, int m, int f, float4 a0, float4 a1,
                                         float4 h4, float4 g4, int len) {
  if constexpr (EPI == EPI_QKV || EPI == EPI_PREFIX) {
    const int rot_rows = (EPI == EPI_QKV ? s.Hq + s.Hkv : s.Hkv) * s.d;
    if (e.rope_cs && f < rot_rows) {
      // two stored pairs -> channels i0, i0 + 1 and i0 + d/2, i0 + d/2 + 1
      const int head = f / s.d, i0 = (f - head * s.d) >> 1;
      int pos;
      bf16* base = rot_head_base<EPI>(s, e, m, head, len, pos);
      rope_turn(e.rope_cs, s.d, pos, i0, a0.x, a0.y);
      rope_turn(e.rope_cs, s.d, pos, i0 + 1, a0.z, a0.w);
      const uint32_t lo = (uint32_t)__bfloat16_as_ushort(f2bf(a0.x)) | ((uint32_t)__bfloat16_as_ushort(f2bf(a0.z)) << 16);
      const uint32_t hi = (uint32_t)__bfloat16_as_ushort(f2bf(a0.y)) | ((uint32_t)__bfloat16_as_ushort(f2bf(a0.w)) << 16);
      *reinterpret_cast<uint32_t*>(base + i0) = lo;
      *reinterpret_cast<uint32_t*>(base + i0 + (s.d >> 1)) = hi;
      return;
    }
  }
  if constexpr (EPI == EPI_PREFIX) {
    const int kvd = s.Hkv * s.d;
    const bool is_v = f >= kvd;
    const int fk = f - (is_v ? kvd : 0);
    const int g = fk / s.d, j = fk - g * s.d;
    store4_bf16(static_cast<bf16*>(is_v ? e.vc : e.kc) +
                    (((size_t)(e.layer * s.Bmax + e.prefix_row) * s.Hkv + g) * s.Ptot + m) * s.d + j,
                a0.x, a0.y, a0.z, a0.w);
    return;
  }
  if constexpr (EPI == EPI_RESID) {
    h4.x = fmaf(g4.x, a0.x, h4.x);
    h4.y = fmaf(g4.y, a0.y, h4.y);
    h4.z = fmaf(g4.z, a0.z, h4.z);
    h4.w = fmaf(g4.w, a0.w, h4.w);
    *reinterpret_cast<float4*>(e.h + (size_t)m * s.D + f) = h4;
  } else if constexpr (EPI == EPI_GEGLU) {
    store4_bf16(static_cast<bf16*>(e.u) + (size_t)m * s.F + f, gelu_tanh_bf16out(a0.x) * a1.x,
                gelu_tanh_bf16out(a0.y) * a1.y, gelu_tanh_bf16out(a0.z) * a1.z, gelu_tanh_bf16out(a0.w) * a1.w);
  } else {
    const int b = m / s.H, t = m - b * s.H;
    const int qd = s.Hq * s.d;
    bf16* dst;
    if (f < qd) {
      const int hq = f / s.d, j = f - hq * s.d;
      dst = static_cast<bf16*>(e.q) + ((size_t)(b * s.Hq + hq) * s.H + t) * s.d + j;
    } else {
      const int kvd = s.Hkv * s.d;
      const bool is_v = f >= qd + kvd;
      const int fk = f - qd - (is_v ? kvd : 0);
      const int g = fk / s.d, j = fk - g * s.d;
      dst = static_cast<bf16*>(is_v ? e.vc : e.kc) +
            (((size_t)(e.layer * s.Bmax + b) * s.Hkv + g) * s.Ptot + len + t) * s.d + j;
    }
    store4_bf16(dst, a0.x, a0.y, a0.z, a0.w);
  }
}

// Two packed int4 codes (nibbles at bits 4i and 16+4i, two's complement)
// -> bf16x2 of code * scale, rounded once (to nearest even).  (n ^ 8) | 0x4300
// is the bf16 of 128 + (code + 8); subtracting 136 is exact.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t w, int i, __nv_bfloat162 sc) {
  const uint32_t t = (((w >> (4 * i)) & 0x000F000Fu) ^ 0x00080008u) | 0x43004300u;
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&t);
  const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
  v = __hmul2(__hsub2(v, off), sc);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int NA, int EPI, bool SPLIT, bool W4, bool NORM>
__global__ void __launch_bounds__(256, 2)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const Shape s,
              const TcPlan p, const TcGemmArgs a) {
  GTRACE_BEGIN();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const TcSmemLayout L = tc_layout(NA, p, W4, NORM);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* a_ready = empty + p.stages;  // int4 weights: A tile dequantised / norm: B tile built
  uint64_t* accf = a_ready + p.stages;
  uint64_t* wfull = accf + 1;  // int4 weights: the packed tile landed (the token tile completes on full)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfull + p.stages);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = blockIdx.x, split = blockIdx.y, ttile = blockIdx.z;
  const int kps = a.K / p.splits;
  const int k0 = split * kps;
  const int nkb = kps / 64;
  const uint32_t ncols = tmem_cols_for(NA * p.tn);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&a_ready[i], 128);
      mbar_init(&wfull[i], 1);
    }
    mbar_init(accf, 1);
    s_flag[0] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Only now, with its TMEM held, may this CTA let the next kernel's CTAs in:
  // a successor that took the TMEM first would wait on us forever.
  pdl_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    // Weight tiles do not depend on the previous kernel: the first ring's worth
    // is requested before waiting for it (programmatic dependent launch).
    // Weights are streamed once per step when one token tile covers the batch;
    // otherwise the other token tiles re-read them from L2.
    const uint64_t pol_w = p.tok_tiles == 1 ? policy_evict_first() : policy_evict_last();
    const int npre = nkb < p.stages ? nkb : p.stages;
    const int wrow = a.w_row0 + ntile * 128 * NA;
    const uint32_t wdst = W4 ? L.a_bytes + L.b_bytes : 0u;         // raw tile or A tile
    const int wx = W4 ? (k0 + 0) / 2 : k0;                            // packed: two codes per byte
    const int wstep = W4 ? 32 : 64;
    // int4 weights: the packed tile completes on its own barrier (wfull), so
    // the dequantising warps turn the first ring into bf16 before the wait;
    // full then counts only the token tile.
    const uint32_t tx = W4 ? L.b_bytes : NORM ? L.a_bytes + L.b_bytes + L.h_bytes : L.a_bytes + L.b_bytes;
    const uint32_t xdst = L.a_bytes;  // the B tile, or (norm) the fp32 staging that the B tile overlays
    for (int kb = 0; kb < npre; ++kb) {
      uint64_t* wbar = W4 ? &wfull[kb] : &full[kb];
      if (W4) mbar_arrive_expect_tx(wbar, L.raw_bytes);
      mbar_arrive_expect_tx(&full[kb], tx);
      tma_load_2d_hint(smem + (size_t)kb * L.stage_bytes + wdst, &tmW, wx + kb * wstep, wrow, wbar, pol_w);
    }
    pdl_wait();
    GTRACE_WAITED();
    for (int kb = 0; kb < npre; ++kb)
      tma_load_2d(smem + (size_t)kb * L.stage_bytes + xdst, &tmX, k0 + kb * 64, ttile * p.tn, &full[kb]);
    int issued = npre;
    for (int kb = npre; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&empty[st], ((kb / p.stages) & 1) ^ 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      uint8_t* sa = smem + (size_t)st * L.stage_bytes;
      uint64_t* wbar = W4 ? &wfull[st] : &full[st];
      if (W4) mbar_arrive_expect_tx(wbar, L.raw_bytes);
      mbar_arrive_expect_tx(&full[st], tx);
      tma_load_2d_hint(sa + wdst, &tmW, wx + kb * wstep, wrow, wbar, pol_w);
      tma_load_2d(sa + xdst, &tmX, k0 + kb * 64, ttile * p.tn, &full[st]);
      issued = kb + 1;
    }
    // Loads still in flight must land before this CTA may exit.
    for (int kb = issued > p.stages ? issued - p.stages : 0; kb < issued; ++kb) {
      if (!mbar_wait(&full[kb % p.stages], (kb / p.stages) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
      if (W4 && !mbar_wait(&wfull[kb % p.stages], (kb / p.stages) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
    }
    GTRACE_MARK(5);  // every load of this CTA has landed
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t idesc = idesc_bf16(128, p.tn);
    for (int kb = 0; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&full[st], (kb / p.stages) & 1, a.err.wait_ns) ||
          ((W4 || NORM) && !mbar_wait(&a_ready[st], (kb / p.stages) & 1, a.err.wait_ns))) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)st * L.stage_bytes);
      const uint64_t a_desc = sw128_desc(sa, 16, 1024);
      const uint64_t b_desc = sw128_desc(sa + L.a_bytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int na = 0; na < NA; ++na)
          umma_bf16(tmem + na * p.tn, desc_add(a_desc, na * 16384u + kk * 32u), desc_add(b_desc, kk * 32u), idesc,
                    (kb | kk) != 0 ? 1u : 0u);
      }
      umma_commit(&empty[st]);  // stage reusable once these MMAs have read it
    }
    umma_commit(accf);  // always issued, so the epilogue wait ends
  } else if (NORM && warp >= 4) {
    // ---------------------------------------------------------------- norm
    // The sum-of-squares slots and the residual stream come from the previous
    // kernel.  rstd for the tile's tokens first (thread = token, two halves of
    // the slots, added in a fixed order), then per K block: thread = (token,
    // 8 features) chunks of the fp32 staging tile -> bf16 y in the swizzled B
    // tile.
    // The scale / shift rows (tables built before the loop) are read before
    // waiting for the previous kernel; a thread's 8 features are the same in
    // every K block (chunk index q = thread % 8), at most two blocks here.
    const int ct = threadIdx.x - 128;
    const int qf = (ct & 7) * 8;
    float4 tc[2][4];
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
      if (kb < nkb) {
        const int kf = k0 + kb * 64 + qf;
        tc[kb][0] = __ldg(reinterpret_cast<const float4*>(a.nscale + kf));
        tc[kb][1] = __ldg(reinterpret_cast<const float4*>(a.nscale + kf + 4));
        tc[kb][2] = __ldg(reinterpret_cast<const float4*>(a.nshift + kf));
        tc[kb][3] = __ldg(reinterpret_cast<const float4*>(a.nshift + kf + 4));
      }
    pdl_wait();
    float* s_rstd = reinterpret_cast<float*>(smem + L.norm_off);
    float* s_part = s_rstd + 64;
    const int mbase = ttile * p.tn;
    {
      // thread = (token j, half): slots half, half + 2, ... with all loads in flight
      const int j = ct & 63, half = ct >> 6;
      float acc = 0.f;
      if (j < p.tn) {
        const float* sp = a.ss_in + mbase + j;
        constexpr int NB = 32;
        for (int s0 = half; s0 < a.nslots; s0 += 2 * NB) {
          float v[NB];
#pragma unroll
          for (int i = 0; i < NB; ++i)
            if (s0 + 2 * i < a.nslots) v[i] = __ldcg(sp + (size_t)(s0 + 2 * i) * a.ss_ld);
#pragma unroll
          for (int i = 0; i < NB; ++i)
            if (s0 + 2 * i < a.nslots) acc += v[i];
        }
      }
      s_part[half * 64 + j] = acc;
      named_bar(3, 128);
      if (ct < 64) s_rstd[ct] = rsqrtf((s_part[ct] + s_part[64 + ct]) / (float)s.D + s.eps);
      named_bar(3, 128);
    }
    for (int kb = 0; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&full[st], (kb / p.stages) & 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      uint8_t* stage = smem + (size_t)st * L.stage_bytes;
      const float* hs = reinterpret_cast<const float*>(stage + L.a_bytes);
      const uint32_t bbase = smem_u32(stage + L.a_bytes);
      float4 c0, c1, d0, d1;
      if (kb == 0) {
        c0 = tc[0][0];
        c1 = tc[0][1];
        d0 = tc[0][2];
        d1 = tc[0][3];
      } else if (kb == 1) {
        c0 = tc[1][0];
        c1 = tc[1][1];
        d0 = tc[1][2];
        d1 = tc[1][3];
      } else {
        const int kf = k0 + kb * 64 + qf;
        c0 = __ldg(reinterpret_cast<const float4*>(a.nscale + kf));
        c1 = __ldg(reinterpret_cast<const float4*>(a.nscale + kf + 4));
        d0 = __ldg(reinterpret_cast<const float4*>(a.nshift + kf));
        d1 = __ldg(reinterpret_cast<const float4*>(a.nshift + kf + 4));
      }
      // thread = (token, 8 features): at most four chunks per thread (tn <= 64)
      uint32_t w[4][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = ct + c * 128;
        if (i < p.tn * 8) {
          const int r = i >> 3;
          const float4 h0 = *reinterpret_cast<const float4*>(hs + r * 64 + qf);
          const float4 h1 = *reinterpret_cast<const float4*>(hs + r * 64 + qf + 4);
          const float rs = s_rstd[r];
          const float y[8] = {h0.x * rs * (1.f + c0.x) + d0.x, h0.y * rs * (1.f + c0.y) + d0.y,
                              h0.z * rs * (1.f + c0.z) + d0.z, h0.w * rs * (1.f + c0.w) + d0.w,
                              h1.x * rs * (1.f + c1.x) + d1.x, h1.y * rs * (1.f + c1.y) + d1.y,
                              h1.z * rs * (1.f + c1.z) + d1.z, h1.w * rs * (1.f + c1.w) + d1.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            w[c][t] = (uint32_t)__bfloat16_as_ushort(f2bf(y[2 * t])) |
                      ((uint32_t)__bfloat16_as_ushort(f2bf(y[2 * t + 1])) << 16);
        }
      }
      named_bar(3, 128);  // every chunk of the staging is read before B overwrites it
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = ct + c * 128;
        if (i < p.tn * 8) {
          const int r = i >> 3, q = i & 7;
          const uint32_t addr = bbase + (uint32_t)r * 128u + (((uint32_t)q ^ (uint32_t)(r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[c][0]), "r"(w[c][1]),
                       "r"(w[c][2]), "r"(w[c][3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&a_ready[st]);
    }
  } else if (W4 && warp >= 4) {
    // ---------------------------------------------------------------- dequant
    // Thread t owns weight row t (and t + 128 for the gate/up pair): its 64
    // packed codes per K block become 64 bf16 code * scale values, written as
    // eight 16-byte chunks in the 128-byte swizzled layout the MMA reads.
    const int dr = threadIdx.x - 128;
    const int gpr = a.K / 128;  // scale groups per weight row
    const bf16* srow0 = a.scales + (size_t)(a.w_row0 + ntile * 128 * NA + dr) * gpr;
    for (int kb = 0; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&wfull[st], (kb / p.stages) & 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      uint8_t* stage = smem + (size_t)st * L.stage_bytes;
      const int g = (k0 + kb * 64) / 128;
#pragma unroll
      for (int na = 0; na < NA; ++na) {
        const int r = dr + na * 128;
        const bf16 sv = srow0[(size_t)na * 128 * gpr + g];
        const __nv_bfloat162 sc = __halves2bfloat162(sv, sv);
        const uint4* raw = reinterpret_cast<const uint4*>(stage + L.a_bytes + L.b_bytes + r * 32);
        const uint4 w0 = raw[0], w1 = raw[1];
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const uint32_t arow = smem_u32(stage) + (uint32_t)r * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = arow + (((uint32_t)c ^ (uint32_t)(r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "r"(dequant_pair(words[c], 0, sc)), "r"(dequant_pair(words[c], 1, sc)),
                       "r"(dequant_pair(words[c], 2, sc)), "r"(dequant_pair(words[c], 3, sc))
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&a_ready[st]);
    }
  }
  __syncwarp();
  pdl_wait();  // the epilogue reads the residual stream / slot lengths

  // ------------------------------------------------------------------ epilogue
  // Factored adaRMSNorm: rstd of the tile's tokens from the producers' sums of
  // squares, while the MMAs finish.  Thread = (token, part): the P parts of a
  // token take every P-th slot with all loads in flight, and the token's
  // thread adds the P partial sums in a fixed order.
  float* s_rs = reinterpret_cast<float*>(smem + L.rs_off);
  constexpr bool kFactor = EPI == EPI_QKV || EPI == EPI_GEGLU;
  if (kFactor && a.e.f_ss) {
    const int P = p.tn <= 64 ? 4 : p.tn <= 128 ? 2 : 1;
    const int col = threadIdx.x % (256 / P), part = threadIdx.x / (256 / P);
    const int m = ttile * p.tn + col;
    if (col < p.tn) {
      float acc = 0.f;
      if (m < a.e.M) {
        const float* sp = a.e.f_ss + m;
        constexpr int NB = 16;
        for (int s0 = part; s0 < a.e.f_nslots; s0 += NB * P) {
          float v[NB];
#pragma unroll
          for (int i = 0; i < NB; ++i)
            v[i] = s0 + i * P < a.e.f_nslots ? __ldcg(sp + (size_t)(s0 + i * P) * a.e.ss_ld) : 0.f;
#pragma unroll
          for (int i = 0; i < NB; ++i) acc += v[i];
        }
      }
      s_rs[part * p.tn + col] = acc;
    }
    __syncthreads();
    if (threadIdx.x < p.tn) {
      float t = 0.f;
      for (int q = 0; q < P; ++q) t += s_rs[q * p.tn + threadIdx.x];
      s_rs[threadIdx.x] = rsqrtf(t / (float)s.D + s.eps);
    }
  }
  const bool acc_ok = mbar_wait(accf, 0, kDrainNs);
  if (!acc_ok) set_error(a.err, DEV_DRAIN);
  GTRACE_MARK(1);  // accumulator complete
  tc_fence_after();
  // CTA-uniform decision: the TMEM loads below are warp-collective.
  const bool ok = __syncthreads_and(acc_ok ? 1 : 0) != 0 && s_flag[0] == 0;

  // Eight epilogue warps: warp w reads TMEM lanes 32*(w%4).. (its rows) and
  // the 16-token chunks c with c % 2 == w / 4.
  const int quarter = warp & 3, half = warp >> 2;
  const int row = quarter * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
  const int mbase = ttile * p.tn;
  const EpiArgs& e = a.e;
  const int nchunks = p.tn / 16;

  if constexpr (!SPLIT) {
    // Per warp, with no barrier across warps: the warp's 32 rows (output
    // features) x 16 tokens of a chunk pass through its own [16][36] fp32 tile
    // (the ring is idle now), thread = row on the way in and thread = (token,
    // 16 consecutive features) on the way out, so each token's 32 features are
    // written as 64 contiguous bytes.  The TMEM load of the warp's next chunk
    // is in flight while the current one is written out.
    constexpr int TLD = 36;  // row stride in floats: 16-byte rows, conflict-free both ways
    float* tb = reinterpret_cast<float*>(smem) + warp * (16 * TLD);
    const int jt = lane >> 1, fh = (lane & 1) * 16;
    const int f = ntile * 128 + quarter * 32 + fh;
    float a0[16], a1[16], b0[16], b1[16];
    auto load = [&](int c, float* x0, float* x1) {
      tmem_ld16(trow + c * 16, x0);
      if (NA == 2) tmem_ld16(trow + p.tn + c * 16, x1);
    };
    auto settle = [&](float* x0, float* x1) {
      tmem_ld_wait();
      reg_fence16(x0);
      if (NA == 2) reg_fence16(x1);
    };
    // factored adaRMSNorm: this thread's row bias (gate/up: the gate row and
    // the up row 128 below it)
    const bool fac = kFactor && e.f_ss != nullptr;
    float fb0 = 0.f, fb1 = 0.f;
    if (fac && ntile * 128 + row < a.N) {
      const int srow = NA == 2 ? ntile * 256 + row : ntile * 128 + row;
      fb0 = e.f_bias[srow];
      if (NA == 2) fb1 = e.f_bias[srow + 128];
    }
    auto emit = [&](int c, const float* x0, const float* x1) {
      if (fac) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float rs = s_rs[c * 16 + j];
          const float g = fmaf(rs, x0[j], fb0);
          tb[j * TLD + lane] = NA == 2 ? gelu_tanh_bf16out(g) * fmaf(rs, x1[j], fb1) : g;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) tb[j * TLD + lane] = NA == 2 ? gelu_tanh_bf16out(x0[j]) * x1[j] : x0[j];
      }
      __syncwarp();
      const int m = mbase + c * 16 + jt;
      if (m < e.M && f < a.N) {
        float v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 t4 = *reinterpret_cast<const float4*>(tb + jt * TLD + fh + 4 * q);
          v[4 * q] = t4.x; v[4 * q + 1] = t4.y; v[4 * q + 2] = t4.z; v[4 * q + 3] = t4.w;
        }
        epi_vec16<EPI>(s, e, m, f, v);
      }
      __syncwarp();
    };
    if (ok) {
      int c = half;
      if (c < nchunks) load(c, a0, a1);
      for (; c < nchunks; c += 4) {
        settle(a0, a1);
        if (c + 2 < nchunks) load(c + 2, b0, b1);
        emit(c, a0, a1);
        if (c + 2 < nchunks) {
          settle(b0, b1);
          if (c + 4 < nchunks) load(c + 4, a0, a1);
          emit(c + 2, b0, b1);
        }
      }
    }
  } else {
    // Split-K inside a cluster of S CTAs: rank r owns rows [r*R, r*R+R).  Every
    // CTA pushes each row's partial into the owner's receive buffer through
    // distributed shared memory (layout [na][src][token][row]); after one
    // cluster barrier each owner sums its rows over the S sources in rank
    // order, reading only local memory, so results are bitwise reproducible
    // and no partial touches global memory.
    const int S = p.splits, R = 128 / S;
    const uint32_t rank = cluster_rank();
    float* recv = reinterpret_cast<float*>(smem + L.recv_off);
    if (p.recv_alias) cluster_sync();  // every peer's MMAs are done with the ring
    if (ok) {
      const int owner = row / R, rr = row - owner * R;
      const uint32_t dst = map_cluster(smem_u32(recv), (uint32_t)owner);
      float a0[16], a1[16], b0[16], b1[16];
      auto load = [&](int c, float* x0, float* x1) {
        tmem_ld16(trow + c * 16, x0);
        if (NA == 2) tmem_ld16(trow + p.tn + c * 16, x1);
      };
      auto settle = [&](float* x0, float* x1) {
        tmem_ld_wait();
        reg_fence16(x0);
        if (NA == 2) reg_fence16(x1);
      };
      auto push = [&](int c, const float* x0, const float* x1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint32_t col = (uint32_t)(c * 16 + j);
          st_cluster_f32(dst + ((((uint32_t)0 * S + rank) * p.tn + col) * R + rr) * 4u, x0[j]);
          if (NA == 2) st_cluster_f32(dst + ((((uint32_t)1 * S + rank) * p.tn + col) * R + rr) * 4u, x1[j]);
        }
      };
      int c = half;
      if (c < nchunks) load(c, a0, a1);
      for (; c < nchunks; c += 4) {
        settle(a0, a1);
        if (c + 2 < nchunks) load(c + 2, b0, b1);
        push(c, a0, a1);
        if (c + 2 < nchunks) {
          settle(b0, b1);
          if (c + 4 < nchunks) load(c + 4, a0, a1);
          push(c + 2, b0, b1);
        }
      }
    }

    // Reduction by thread = (4 consecutive rows of this rank, token): rows
    // 4*(t % (R/4)).. and tokens t / (R/4) + k * 256 / (R/4), one float4 per
    // source in rank order.  The loads the epilogue needs (residual stream,
    // gate, slot lengths) are issued before the cluster barrier, so they
    // overlap the wait for the slowest rank.  The residual epilogue that also
    // feeds the next norm (ss_out) adds the squares of a token's R rows over
    // its R/4 adjacent lanes into slot (tile * S + rank).
    constexpr int UB = 8;  // tokens per batch
    constexpr bool vec = true;
    const int G4 = R / 4, lg4 = __ffs(G4) - 1;
    const int g4 = threadIdx.x & (G4 - 1);
    const int cstep4 = 256 >> lg4;
    const int col0 = threadIdx.x >> lg4;
    const int fv = ntile * 128 + (int)rank * R + 4 * g4;
    const bool fv_ok = fv < a.N;
    const bool need_len = EPI == EPI_QKV && (fv >= s.Hq * s.d || e.rope_cs);
    float4 hv[UB];
    int lv[UB];
    float4 gv = make_float4(0.f, 0.f, 0.f, 0.f), ysv = gv;
    if (EPI == EPI_RESID && ok && vec && fv_ok) {
      gv = *reinterpret_cast<const float4*>(e.gate + fv);
      if (e.y_out) ysv = *reinterpret_cast<const float4*>(e.y_scale + fv);
    }
    // factored adaRMSNorm: the 4 rows' bias (gate/up: gate rows, up rows 128 below)
    const bool fac = kFactor && e.f_ss != nullptr;
    float4 fbv0 = make_float4(0.f, 0.f, 0.f, 0.f), fbv1 = fbv0;
    if (fac && ok && fv_ok) {
      const int srow = NA == 2 ? ntile * 256 + (fv - ntile * 128) : fv;
      fbv0 = *reinterpret_cast<const float4*>(e.f_bias + srow);
      if (NA == 2) fbv1 = *reinterpret_cast<const float4*>(e.f_bias + srow + 128);
    }
    auto prefetch = [&](int cb) {
#pragma unroll
      for (int k = 0; k < UB; ++k) {
        const int col = cb + k * cstep4, m = mbase + col;
        if (col < p.tn && m < e.M && fv_ok) {
          if constexpr (EPI == EPI_RESID) hv[k] = __ldcg(reinterpret_cast<const float4*>(e.h + (size_t)m * s.D + fv));
          if constexpr (EPI == EPI_QKV) lv[k] = need_len ? e.lens[m / s.H] : 0;
        }
      }
    };
    GTRACE_MARK(2);  // partials pushed
    if (ok && vec) prefetch(col0);
    cluster_sync();
    GTRACE_MARK(3);  // every rank's partials arrived
    if (ok && vec) {
      const uint32_t rb = smem_u32(recv) + (uint32_t)(16 * g4);
      const uint32_t src_stride = (uint32_t)p.tn * R * 4u;
      const uint32_t na_stride = (uint32_t)S * src_stride;
#pragma unroll 1
      for (int cb = col0; cb < p.tn; cb += UB * cstep4) {
        if (cb != col0) prefetch(cb);
        float4 s0[UB], s1[UB];
#pragma unroll
        for (int k = 0; k < UB; ++k) {
          s0[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          s1[k] = s0[k];
        }
#pragma unroll 1
        for (int src = 0; src < S; ++src) {
#pragma unroll
          for (int k = 0; k < UB; ++k) {
            const int col = cb + k * cstep4;
            if (col < p.tn) {
              const uint32_t addr = rb + (uint32_t)col * R * 4u + (uint32_t)src * src_stride;
              add4(s0[k], ld_shared_f32x4(addr));
              if (NA == 2) add4(s1[k], ld_shared_f32x4(addr + na_stride));
            }
          }
        }
#pragma unroll
        for (int k = 0; k < UB; ++k) {
          const int col = cb + k * cstep4, m = mbase + col;
          if (col < p.tn && m < e.M && fv_ok) {
            if (fac) {
              const float rs = s_rs[col];
              s0[k] = make_float4(fmaf(rs, s0[k].x, fbv0.x), fmaf(rs, s0[k].y, fbv0.y), fmaf(rs, s0[k].z, fbv0.z),
                                  fmaf(rs, s0[k].w, fbv0.w));
              if (NA == 2)
                s1[k] = make_float4(fmaf(rs, s1[k].x, fbv1.x), fmaf(rs, s1[k].y, fbv1.y), fmaf(rs, s1[k].z, fbv1.z),
                                    fmaf(rs, s1[k].w, fbv1.w));
            }
            epi_vec4<EPI>(s, e, m, fv, s0[k], s1[k], hv[k], gv, lv[k]);
          }
        }
        if constexpr (EPI == EPI_RESID) {
          if (e.ss_out) {
            // the next norm: operand bf16(h (1 + scale)) of the 4 rows, and the
            // sum of squares of h over this rank's R rows per token (the R/4
            // threads of a token are adjacent lanes: fixed shuffle tree)
#pragma unroll
            for (int k = 0; k < UB; ++k) {
              const int col = cb + k * cstep4, m = mbase + col;
              const bool valid = col < p.tn && m < e.M && fv_ok;
              float sq = 0.f;
              if (valid) {
                const float4 h4 = make_float4(fmaf(gv.x, s0[k].x, hv[k].x), fmaf(gv.y, s0[k].y, hv[k].y),
                                              fmaf(gv.z, s0[k].z, hv[k].z), fmaf(gv.w, s0[k].w, hv[k].w));
                sq = fmaf(h4.x, h4.x, fmaf(h4.y, h4.y, fmaf(h4.z, h4.z, h4.w * h4.w)));
                if (e.y_out)
                  store4_bf16(static_cast<bf16*>(e.y_out) + (size_t)m * s.D + fv, h4.x * (1.f + ysv.x),
                              h4.y * (1.f + ysv.y), h4.z * (1.f + ysv.z), h4.w * (1.f + ysv.w));
              }
              const unsigned gm = G4 >= 32 ? 0xffffffffu : (((1u << G4) - 1u) << (lane & ~(G4 - 1)));
              for (int o = 1; o < G4; o <<= 1) sq += __shfl_xor_sync(gm, sq, o);
              if (valid && g4 == 0) e.ss_out[(size_t)(ntile * S + (int)rank) * e.ss_ld + m] = sq;
            }
          }
        }
      }
    }
  }

  GTRACE_MARK(4);  // epilogue written
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
  GTRACE_END(1 + EPI);
}

size_t smem_bytes_impl(int na, const TcPlan& p, bool w4, bool norm) { return tc_layout(na, p, w4, norm).total; }

template <int NA, int EPI, bool SPLIT, bool W4, bool NORM>
cudaError_t init_one() {
  auto kern = k_tc_gemm<NA, EPI, SPLIT, W4, NORM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess && SPLIT) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int NA, int EPI, bool W4, bool NORM>
cudaError_t launch_one(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, const TcPlan& p,
                       const TcGemmArgs& a, bool pdl, cudaStream_t st) {
  dim3 grid((a.N + 127) / 128, p.splits, p.tok_tiles);
  const size_t smem = smem_bytes_impl(NA, p, W4, NORM);
  if (p.splits > 1)
    return launch_ex(k_tc_gemm<NA, EPI, true, W4, NORM>, grid, dim3(256), smem, st, p.splits, pdl, *tmW, *tmX, s, p,
                     a);
  return launch_ex(k_tc_gemm<NA, EPI, false, W4, NORM>, grid, dim3(256), smem, st, 1, pdl, *tmW, *tmX, s, p, a);
}

template <bool W4>
cudaError_t init_all() {
  cudaError_t e = init_one<1, EPI_QKV, false, W4, false>();
  if (e == cudaSuccess) e = init_one<1, EPI_QKV, true, W4, false>();
  if (e == cudaSuccess) e = init_one<1, EPI_RESID, false, W4, false>();
  if (e == cudaSuccess) e = init_one<1, EPI_RESID, true, W4, false>();
  if (e == cudaSuccess) e = init_one<2, EPI_GEGLU, false, W4, false>();
  if (e == cudaSuccess) e = init_one<2, EPI_GEGLU, true, W4, false>();
  return e;
}

cudaError_t init_prefix() {
  cudaError_t e = init_one<1, EPI_PREFIX, false, false, false>();
  if (e == cudaSuccess) e = init_one<1, EPI_PREFIX, true, false, false>();
  return e;
}

cudaError_t init_norm() {
  cudaError_t e = init_one<1, EPI_QKV, false, false, true>();
  if (e == cudaSuccess) e = init_one<1, EPI_QKV, true, false, true>();
  if (e == cudaSuccess) e = init_one<2, EPI_GEGLU, false, false, true>();
  if (e == cudaSuccess) e = init_one<2, EPI_GEGLU, true, false, true>();
  return e;
}

template <bool W4>
cudaError_t launch_sel(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, int na, const TcPlan& p,
                       const TcGemmArgs& a, bool pdl, cudaStream_t st) {
  if (na == 2) return launch_one<2, EPI_GEGLU, W4, false>(s, tmW, tmX, p, a, pdl, st);
  if (a.e.epi == EPI_QKV) return launch_one<1, EPI_QKV, W4, false>(s, tmW, tmX, p, a, pdl, st);
  return launch_one<1, EPI_RESID, W4, false>(s, tmW, tmX, p, a, pdl, st);
}

}  // namespace

size_t tc_gemm_smem_bytes(int na, const TcPlan& p, bool w4, bool norm) { return smem_bytes_impl(na, p, w4, norm); }

cudaError_t tc_gemm_init() {
  cudaError_t e = init_all<false>();
  if (e == cudaSuccess) e = init_all<true>();
  if (e == cudaSuccess) e = init_norm();
  if (e == cudaSuccess) e = init_prefix();
  return e;
}

cudaError_t launch_tc_gemm(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, int na, const TcPlan& p,
                           const TcGemmArgs& a, bool pdl, cudaStream_t st) {
  if (a.e.epi == EPI_PREFIX) {  // prefix production: bf16 weights, keys/values into the slots
    if (a.scales || a.ss_in || na != 1) return cudaErrorInvalidValue;
    return launch_one<1, EPI_PREFIX, false, false>(s, tmW, tmX, p, a, pdl, st);
  }
  if (a.ss_in) {  // adaRMSNorm in the kernel: bf16 weights only, QKV or gate/up
    if (a.scales) return cudaErrorInvalidValue;
    if (na == 2) return launch_one<2, EPI_GEGLU, false, true>(s, tmW, tmX, p, a, pdl, st);
    if (a.e.epi != EPI_QKV) return cudaErrorInvalidValue;
    return launch_one<1, EPI_QKV, false, true>(s, tmW, tmX, p, a, pdl, st);
  }
  if (a.scales) return launch_sel<true>(s, tmW, tmX, na, p, a, pdl, st);
  return launch_sel<false>(s, tmW, tmX, na, p, a, pdl, st);
}

}  // namespace pae

#ifdef PAE_GRAPH_TRACE
// Trace builds only: hand this file's kernels the launch-trace buffer.
extern "C" int pae_graph_trace_bind_gemm(void* buf, void* ctr, unsigned cap) {
  return (int)pae::gtrace_bind_tu(buf, ctr, cap);
}
#endif
