// prologue.cuh -- per-head Q/K RMSNorm + rotary position embedding.
//
// The fused norm/RoPE step that feeds attention in the MiniMax-H3 DiT block
// ("H3 Runtime Current State", Owned Performance Kernels: fused Q/K RMSNorm,
// RoPE and layout work; "Buyer Questions: Current Evidence Status", block composition: norm/RoPE
// share of the block).  The operation is stated in h3attn.h (h3attn_prologue).
//
// Work layout: one warp per token.  A row of head_dim bf16 values is 16 lanes x
// 16 bytes (d = 128) or 8 lanes x 16 bytes (d = 64), so one warp pass covers
// (Q_h, K_h) for d = 128 or (Q_h, K_h, Q_h+1, K_h+1) for d = 64.  Loads and
// stores are 128-bit and coalesced per row; the sum of squares is a shuffle
// reduction inside each row's lane group; a lane owns whole rotation pairs, so
// RoPE needs no data exchange.  The cos/sin of the token's pairs are computed
// once per token in fp64 and reused by every head of Q and K.
//
// Precision: x*gamma is exact in fp32 (8-bit x 8-bit significands) and the
// RMS scale factor r multiplies a whole row, so it only adds a relative error.
// The rotation of a = x*gamma is the complex product a*c + (-a1, a0)*s with
// cos and sin from fp64 carried as float pairs (hi + lo): the sine term's hi
// product is split into its rounded value and exact error (fma), so the one
// rounded sum a*c_hi + q is within 2^-24 of the result even where the two terms
// cancel, and the small terms carry the rest.  The result is therefore within a
// few fp32 ulps (relative) of the exact value, i.e. within one bf16 ulp of its
// correctly rounded bf16.  Pairs of elements go through packed fp32 arithmetic
// (two values per instruction), which halves the instructions the rotation and
// the norm issue; three 256-thread blocks stay resident per SM.  The kernel is
// HBM-bound: two reads and two writes of n_tokens * n_heads * d bf16 values.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "common.cuh"

namespace h3 {

constexpr int kRopeMaxPairs = 64;

// Per-pair rotary tables, computed on the host in double precision.
struct RopeTables {
  double inv_freq_3d[kRopeMaxPairs];  // theta^(-2i/ds) of pair p inside its section
  double inv_freq_1d[kRopeMaxPairs];  // theta^(-2p/d)
  uint8_t axis_3d[kRopeMaxPairs];     // 0 = t, 1 = h, 2 = w
};

struct PrologueParams {
  const uint16_t* q_in;
  const uint16_t* k_in;
  uint16_t* q_out;
  uint16_t* k_out;
  int64_t n_tokens;
  int64_t in_tok, in_head, out_tok, out_head;  // element strides
  const uint16_t* gamma_q;                     // may be null
  const uint16_t* gamma_k;                     // may be null
  const int32_t* pos;                          // may be null
  const uint8_t* kind;
  int32_t n_heads;
  float eps;
  RopeTables rope;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&y)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = ptx::pack_bf16x2(y[2 * i], y[2 * i + 1]);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D>
__global__ void __launch_bounds__(256, 3) prologue_kernel(const __grid_constant__ PrologueParams p) {
  constexpr int kRowLanes = D / 8;             // lanes per row (16 B each)
  constexpr int kRowsPerPass = 32 / kRowLanes;  // rows per warp pass (Q/K interleaved)
  constexpr int kHeadsPerPass = kRowsPerPass / 2;
  constexpr int kUnroll = 4;

  const int lane = threadIdx.x & 31;
  const int64_t token = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (token >= p.n_tokens) return;

  const int group = lane / kRowLanes;     // which row of the pass
  const int chunk = lane % kRowLanes;     // which 8 elements of the row
  const bool is_k = (group & 1) != 0;
  const int head_in_pass = group >> 1;

  const uint16_t* src = is_k ? p.k_in : p.q_in;
  uint16_t* dst = is_k ? p.k_out : p.q_out;
  const uint16_t* gamma = is_k ? p.gamma_k : p.gamma_q;

  // gamma of this lane's 8 elements (fp32, exact)
  float g[8];
  const bool do_norm = gamma != nullptr;
  const bool any_norm = p.gamma_q != nullptr || p.gamma_k != nullptr;
  if (do_norm) {
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(gamma + chunk * 8), g);
  }

  // cos/sin of this lane's 4 pairs for this token (fp64)
  int kind = 0;
  int32_t pt = 0, ph = 0, pw = 0;
  if (p.pos != nullptr) {
    kind = p.kind[token];
    if (kind == 1 || kind == 2) {
      pt = p.pos[3 * token + 0];
      ph = p.pos[3 * token + 1];
      pw = p.pos[3 * token + 2];
    } else {
      kind = 0;
    }
  }
  const bool do_rope = kind != 0;
  // cos and sin as unevaluated float pairs (hi + lo, |lo| <= ulp(hi)/2): the
  // rotation below then runs in fp32 with error-free products, avoiding per-element
  // fp32 <-> fp64 conversions (which share the slow conversion pipe).
  float ch[4], cl[4], sh[4], sl[4];
  if (do_rope) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int pair = chunk * 4 + k;
      double angle;
      if (kind == 1) {
        const int ax = p.rope.axis_3d[pair];
        const int32_t pp = ax == 0 ? pt : (ax == 1 ? ph : pw);
        angle = static_cast<double>(pp) * p.rope.inv_freq_3d[pair];
      } else {
        angle = static_cast<double>(pt) * p.rope.inv_freq_1d[pair];
      }
      double sd, cd;
      sincos(angle, &sd, &cd);
      ch[k] = static_cast<float>(cd);
      cl[k] = static_cast<float>(cd - static_cast<double>(ch[k]));
      sh[k] = static_cast<float>(sd);
      sl[k] = static_cast<float>(sd - static_cast<double>(sh[k]));
    }
  }

  const float inv_d = 1.0f / static_cast<float>(D);
  const int n_heads = p.n_heads;
  const int n_pass = (n_heads + kHeadsPerPass - 1) / kHeadsPerPass;

  for (int pass0 = 0; pass0 < n_pass; pass0 += kUnroll) {
    uint4 raw[kUnroll];
    bool live[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int h = (pass0 + u) * kHeadsPerPass + head_in_pass;
      live[u] = (pass0 + u) < n_pass && h < n_heads;
      if (live[u]) {
        raw[u] = *reinterpret_cast<const uint4*>(src + token * p.in_tok + h * p.in_head + chunk * 8);
      } else {
        raw[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float x[8];
      bf16x8_to_f32(raw[u], x);
      float r = 1.0f;
      if (any_norm) {  // warp-uniform: every lane joins the shuffles
        float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 xi = make_float2(x[2 * i], x[2 * i + 1]);
          ss2 = __ffma2_rn(xi, xi, ss2);
        }
        float ss = ss2.x + ss2.y;
#pragma unroll
        for (int off = kRowLanes / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (do_norm) {
          r = rsqrtf(fmaf(ss, inv_d, p.eps));
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // exact
            const float2 xg = __fmul2_rn(make_float2(x[2 * i], x[2 * i + 1]), make_float2(g[2 * i], g[2 * i + 1]));
            x[2 * i] = xg.x;
            x[2 * i + 1] = xg.y;
          }
        }
      }
      float y[8];
      if (do_rope) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // The pair a = (a0, a1) = x*gamma is exact in fp32.  As a complex product,
          // y = a*c + ra*s with ra = (-a1, a0) and c, s each an unevaluated float pair
          // (hi + lo).  The sine term's hi product is split into its rounded value q
          // and exact error e (fma); m = a*c_hi + q then rounds once to within 2^-24
          // of the result even where the two terms cancel, and the small terms
          // (e, a*c_lo, ra*s_lo) carry the rest.  Each line works on both elements of
          // the pair at once (packed fp32 pairs).
          const float2 a = make_float2(x[2 * k], x[2 * k + 1]);
          const float2 ra = make_float2(-x[2 * k + 1], x[2 * k]);
          const float2 shi = make_float2(sh[k], sh[k]), slo = make_float2(sl[k], sl[k]);
          const float2 chi = make_float2(ch[k], ch[k]), clo = make_float2(cl[k], cl[k]);
          const float2 q = __fmul2_rn(ra, shi);
          const float2 e = __ffma2_rn(ra, shi, make_float2(-q.x, -q.y));
          const float2 m = __ffma2_rn(a, chi, q);
          float2 lo = __ffma2_rn(a, clo, e);
          lo = __ffma2_rn(ra, slo, lo);
          const float2 yy = __fmul2_rn(__fadd2_rn(m, lo), make_float2(r, r));
          y[2 * k] = yy.x;
          y[2 * k + 1] = yy.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[i] * r;
      }
      const int h = (pass0 + u) * kHeadsPerPass + head_in_pass;
      if (live[u] && store_in_bounds(token < p.n_tokens && h < n_heads && chunk * 8 + 8 <= D)) {
        *reinterpret_cast<uint4*>(dst + token * p.out_tok + h * p.out_head + chunk * 8) =
            f32x8_to_bf16(y);
      }
    }
  }
}

}  // namespace h3
