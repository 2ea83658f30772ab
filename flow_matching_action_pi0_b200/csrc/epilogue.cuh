// GEMM epilogues shared by the CUDA-core and tcgen05 projection kernels.
// One call handles one (token m, output feature f) with the accumulated
// dot products acc0 (and acc1 for the GeGLU up projection).
#pragma once

#include "internal.h"

namespace pae {

// [q | k | v] = y W_qkv^T: q goes to the per-request head-major buffer
// q[b][hq][i][:], k and v into this layer's KV slot of request b right after its
// prefix (position lens[b] + i), so attention reads one contiguous key range.
template <typename TA>
__device__ __forceinline__ void epi_qkv(const Shape& s, const EpiArgs& e, int m, int f, float acc) {
  const int b = m / s.H, i = m - b * s.H;
  const int qd = s.Hq * s.d;
  if (f < qd) {
    const int hq = f / s.d, j = f - hq * s.d;
    st_act<TA>(static_cast<TA*>(e.q) + ((size_t)(b * s.Hq + hq) * s.H + i) * s.d + j, acc);
  } else {
    const int kvd = s.Hkv * s.d;
    const bool is_v = f >= qd + kvd;
    const int fk = f - qd - (is_v ? kvd : 0);
    const int g = fk / s.d, j = fk - g * s.d;
    const int pos = e.lens[b] + i;
    const size_t off = (((size_t)(e.layer * s.Bmax + b) * s.Hkv + g) * s.Ptot + pos) * s.d + j;
    st_act<TA>(static_cast<TA*>(is_v ? e.vc : e.kc) + off, acc);
  }
}

// Rotary embedding: inside every rotated head (the q heads, then the k heads)
// the projection rows are stored pair-interleaved, row 2i = channel i and row
// 2i + 1 = channel i + d/2, so both members of a rotated pair leave the GEMM
// side by side.  Channel of the (head-local) stored row p:
__host__ __device__ __forceinline__ int rope_channel(int p, int d) { return (p >> 1) + (p & 1) * (d >> 1); }

// Turn the pair (a = channel i, b = channel i + d/2) by the tabled angle of
// position pos: a' = a cos - b sin, b' = b cos + a sin.
__device__ __forceinline__ void rope_turn(const float2* cs, int d, int pos, int i, float& a, float& b) {
  const float2 t = cs[(size_t)pos * (d >> 1) + i];
  const float x = a * t.x - b * t.y;
  const float y = b * t.x + a * t.y;
  a = x;
  b = y;
}

// One stored pair (even row f, f + 1) of the q/k block with rotation: both
// results land on their natural channels.
template <typename TA>
__device__ __forceinline__ void epi_qkv_pair(const Shape& s, const EpiArgs& e, int m, int f, float a0, float a1) {
  const int rot_rows = (s.Hq + s.Hkv) * s.d;
  if (!e.rope_cs || f >= rot_rows) {
    epi_qkv<TA>(s, e, m, f, a0);
    epi_qkv<TA>(s, e, m, f + 1, a1);
    return;
  }
  const int b = m / s.H, t = m - b * s.H;
  const int head = f / s.d, i = (f - head * s.d) >> 1;
  rope_turn(e.rope_cs, s.d, e.lens[b] + t, i, a0, a1);
  epi_qkv<TA>(s, e, m, head * s.d + i, a0);
  epi_qkv<TA>(s, e, m, head * s.d + i + (s.d >> 1), a1);
}

// Prefix production: token m is position m of request e.prefix_row; output
// features [0, Hkv d) are its keys (rotated at position m when rope is on,
// rows pair-interleaved like the q/k block), [Hkv d, 2 Hkv d) its values.
template <typename TA>
__device__ __forceinline__ void epi_prefix(const Shape& s, const EpiArgs& e, int m, int f, float acc) {
  const int kvd = s.Hkv * s.d;
  const bool is_v = f >= kvd;
  const int fk = f - (is_v ? kvd : 0);
  const int g = fk / s.d, j = fk - g * s.d;
  const size_t off = (((size_t)(e.layer * s.Bmax + e.prefix_row) * s.Hkv + g) * s.Ptot + m) * s.d + j;
  st_act<TA>(static_cast<TA*>(is_v ? e.vc : e.kc) + off, acc);
}
template <typename TA>
__device__ __forceinline__ void epi_prefix_pair(const Shape& s, const EpiArgs& e, int m, int f, float a0, float a1) {
  const int kvd = s.Hkv * s.d;
  if (!e.rope_cs || f >= kvd) {
    epi_prefix<TA>(s, e, m, f, a0);
    epi_prefix<TA>(s, e, m, f + 1, a1);
    return;
  }
  const int head = f / s.d, i = (f - head * s.d) >> 1;
  rope_turn(e.rope_cs, s.d, m, i, a0, a1);
  epi_prefix<TA>(s, e, m, head * s.d + i, a0);
  epi_prefix<TA>(s, e, m, head * s.d + i + (s.d >> 1), a1);
}

// h += gate * acc  (gated residual; gate from this step's modulation table)
__device__ __forceinline__ void epi_resid(const Shape& s, const EpiArgs& e, int m, int f, float acc) {
  float* hp = e.h + (size_t)m * s.D + f;
  *hp = fmaf(e.gate[f], acc, *hp);
}

// u = gelu_tanh(y W_gate^T) * (y W_up^T)
template <typename TA>
__device__ __forceinline__ void epi_geglu(const Shape& s, const EpiArgs& e, int m, int f, float g, float up) {
  if constexpr (sizeof(TA) == 2)
    st_act<TA>(static_cast<TA*>(e.u) + (size_t)m * s.F + f, gelu_tanh_bf16out(g) * up);
  else
    st_act<TA>(static_cast<TA*>(e.u) + (size_t)m * s.F + f, gelu_tanh(g) * up);
}

template <typename TA>
__device__ __forceinline__ void epi_apply(const Shape& s, const EpiArgs& e, int m, int f, float a0, float a1) {
  if (e.epi == EPI_QKV)
    epi_qkv<TA>(s, e, m, f, a0);
  else if (e.epi == EPI_RESID)
    epi_resid(s, e, m, f, a0);
  else
    epi_geglu<TA>(s, e, m, f, a0, a1);
}

// Row of the weight matrix holding output feature f (GeGLU: gate/up
// interleaved in 128-row tiles: tile t = [gate rows 128t.., up rows 128t..]).
__host__ __device__ __forceinline__ int gate_row(int f) { return (f >> 7) * 256 + (f & 127); }

}  // namespace pae
