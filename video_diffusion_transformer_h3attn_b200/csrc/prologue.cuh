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
// the rotation itself needs no data exchange.  The cos/sin of the token's pairs
// are computed once per token in fp64 (each pair by one of the lanes that share
// it, then handed round by shuffles) and reused by every head of Q and K.  The
// rows reach the warp through a per-warp ring in shared memory filled by 16-byte
// cp.async copies several passes ahead, so many rows are in flight per warp
// without holding registers for them.
//
// Precision: x*gamma is exact in fp32 (8-bit x 8-bit significands) and the
// RMS scale factor r multiplies a whole row, so it only adds a relative error.
// The rotation of (a0, a1) = x*gamma is y0 = a0*c - a1*s, y1 = a1*c + a0*s with
// cos and sin from fp64 carried as float pairs (hi + lo): the sine term's hi
// product is split into its rounded value q and exact error (fma), so the one
// rounded sum (cosine term's hi product) + q is within 2^-24 of the result even
// where the two terms cancel, and the small terms carry the rest.  The result is therefore within a
// few fp32 ulps (relative) of the exact value, i.e. within one bf16 ulp of its
// correctly rounded bf16.  The arithmetic runs in packed fp32 pairs (two values
// per instruction), each pair holding the same position of two neighbouring
// rotation pairs, so the cos/sin of those two pairs are packed alike and no
// operand has to be duplicated or swapped per pass; four 256-thread blocks stay
// resident per SM (64 registers, 32 KB of ring each).  The kernel is HBM-bound:
// two reads and two writes of n_tokens * n_heads * d bf16 values.
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

// 8 bf16 values (elements 0..7 = pairs 0..3) as two couples of pairs: a0[j] = the
// first elements of pairs 2j, 2j+1; a1[j] = their second elements.
__device__ __forceinline__ void bf16x8_to_couples(const uint4& u, float2 (&a0)[2], float2 (&a1)[2]) {
  a0[0] = make_float2(__uint_as_float(u.x << 16), __uint_as_float(u.y << 16));
  a1[0] = make_float2(__uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y & 0xFFFF0000u));
  a0[1] = make_float2(__uint_as_float(u.z << 16), __uint_as_float(u.w << 16));
  a1[1] = make_float2(__uint_as_float(u.z & 0xFFFF0000u), __uint_as_float(u.w & 0xFFFF0000u));
}

// 16-byte asynchronous global -> shared copy (bypasses the register file and L1).
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kPrologueThreads = 256;
constexpr int kPrologueDepth = 8;  // passes in flight per warp

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4) prologue_kernel(const __grid_constant__ PrologueParams p) {
  constexpr int kRowLanes = D / 8;              // lanes per row (16 B each)
  constexpr int kRowsPerPass = 32 / kRowLanes;  // rows per warp pass (Q/K interleaved)
  constexpr int kHeadsPerPass = kRowsPerPass / 2;
  constexpr int kPairsPerLane = 4 / kRowsPerPass;  // sincos each lane evaluates (of its chunk's 4 pairs)
  constexpr int kWarps = kPrologueThreads / 32;
  // Each warp streams its token's rows through a ring of kPrologueDepth passes in shared
  // memory (one 16-byte slot per lane and pass): a lane copies and later reads only its own
  // slot, so its own cp.async groups order the ring and no barrier is needed.
  __shared__ uint4 ring[kWarps][kPrologueDepth][32];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t token = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  if (token >= p.n_tokens) return;

  const int group = lane / kRowLanes;     // which row of the pass
  const int chunk = lane % kRowLanes;     // which 8 elements of the row
  const bool is_k = (group & 1) != 0;
  const int head_in_pass = group >> 1;

  const uint16_t* src = (is_k ? p.k_in : p.q_in) + token * p.in_tok + chunk * 8;
  uint16_t* dst = (is_k ? p.k_out : p.q_out) + token * p.out_tok + chunk * 8;
  const uint16_t* gamma = is_k ? p.gamma_k : p.gamma_q;
  const int n_heads = p.n_heads;
  const int n_pass = (n_heads + kHeadsPerPass - 1) / kHeadsPerPass;

  // The first passes' rows are in flight while the token's angles are evaluated.
#pragma unroll
  for (int s = 0; s < kPrologueDepth; ++s) {
    const int h = s * kHeadsPerPass + head_in_pass;
    if (s < n_pass && h < n_heads) cp_async16(&ring[warp][s][lane], src + h * p.in_head);
    cp_async_commit();
  }

  // The lane's 8 elements as two couples of rotation pairs: couple j holds pairs
  // 2j and 2j+1, a0 = (first elements of both pairs), a1 = (second elements), so
  // one packed fp32 instruction works on the same position of two pairs and the
  // pairs' cos/sin come packed the same way.
  // gamma of this lane's 8 elements (fp32, exact), in couples
  float2 g0[2], g1[2];
  const bool do_norm = gamma != nullptr;
  const bool any_norm = p.gamma_q != nullptr || p.gamma_k != nullptr;
  if (do_norm) {
    const uint4 gw = *reinterpret_cast<const uint4*>(gamma + chunk * 8);
    bf16x8_to_couples(gw, g0, g1);
  }

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
  const bool do_rope = kind != 0;  // warp-uniform (one token per warp)
  // cos and sin of this lane's 4 rotation pairs as unevaluated float pairs (hi + lo,
  // |lo| <= ulp(hi)/2), from fp64: the rotation below then runs in fp32 with error-free
  // products.  The kRowsPerPass lanes that share a chunk need the same 4 pairs, so each
  // evaluates kPairsPerLane of them and the four values per pair are exchanged by shuffles.
  float2 chi[2], clo[2], shi[2], slo[2];
  if (do_rope) {
    float mch[kPairsPerLane], mcl[kPairsPerLane], msh[kPairsPerLane], msl[kPairsPerLane];
#pragma unroll
    for (int k = 0; k < kPairsPerLane; ++k) {
      const int pair = chunk * 4 + group * kPairsPerLane + k;
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
      mch[k] = static_cast<float>(cd);
      mcl[k] = static_cast<float>(cd - static_cast<double>(mch[k]));
      msh[k] = static_cast<float>(sd);
      msl[k] = static_cast<float>(sd - static_cast<double>(msh[k]));
    }
    float ch[4], cl[4], sh[4], sl[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int from = (k / kPairsPerLane) * kRowLanes + chunk;  // the lane that evaluated pair chunk*4+k
      ch[k] = __shfl_sync(0xffffffffu, mch[k % kPairsPerLane], from);
      cl[k] = __shfl_sync(0xffffffffu, mcl[k % kPairsPerLane], from);
      sh[k] = __shfl_sync(0xffffffffu, msh[k % kPairsPerLane], from);
      sl[k] = __shfl_sync(0xffffffffu, msl[k % kPairsPerLane], from);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      chi[j] = make_float2(ch[2 * j], ch[2 * j + 1]);
      clo[j] = make_float2(cl[2 * j], cl[2 * j + 1]);
      shi[j] = make_float2(sh[2 * j], sh[2 * j + 1]);
      slo[j] = make_float2(sl[2 * j], sl[2 * j + 1]);
    }
  }

  const float inv_d = 1.0f / static_cast<float>(D);
  const int64_t in_step = static_cast<int64_t>(kHeadsPerPass) * p.in_head;
  const int64_t out_step = static_cast<int64_t>(kHeadsPerPass) * p.out_head;
  const uint16_t* refill = src + head_in_pass * p.in_head + kPrologueDepth * in_step;  // pass + kPrologueDepth
  uint16_t* out = dst + head_in_pass * p.out_head;
  int h = head_in_pass;
  for (int pass = 0; pass < n_pass; ++pass, h += kHeadsPerPass, refill += in_step, out += out_step) {
    const int slot = pass % kPrologueDepth;
    const bool live = h < n_heads;
    cp_async_wait<kPrologueDepth - 1>();  // this pass's group has landed
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (live) raw = ring[warp][slot][lane];

    float2 a0[2], a1[2];
    bf16x8_to_couples(raw, a0, a1);
    float r = 1.0f;
    if (any_norm) {  // warp-uniform: every lane joins the shuffles
      float2 ss2 = __fmul2_rn(a0[0], a0[0]);
      ss2 = __ffma2_rn(a1[0], a1[0], ss2);
      ss2 = __ffma2_rn(a0[1], a0[1], ss2);
      ss2 = __ffma2_rn(a1[1], a1[1], ss2);
      float ss = ss2.x + ss2.y;
#pragma unroll
      for (int off = kRowLanes / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (do_norm) {
        r = rsqrtf(fmaf(ss, inv_d, p.eps));
#pragma unroll
        for (int j = 0; j < 2; ++j) {  // exact
          a0[j] = __fmul2_rn(a0[j], g0[j]);
          a1[j] = __fmul2_rn(a1[j], g1[j]);
        }
      }
    }
    const float2 rr = make_float2(r, r);
    float2 y0[2], y1[2];
    if (do_rope) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        // Each pair (a0, a1) = x*gamma is exact in fp32; its rotation is
        //   y0 = a0*c - a1*s,  y1 = a1*c + a0*s,
        // with c, s each an unevaluated float pair (hi + lo).  In each line the
        // sine term's hi product is split into its rounded value q and exact error e
        // (fma); m = (cosine term's hi product) + q then rounds once to within 2^-24
        // of the result even where the two terms cancel, and the small terms (e and
        // the lo products) carry the rest.
        const float2 q0 = __fmul2_rn(a1[j], shi[j]);
        const float2 nq0 = make_float2(-q0.x, -q0.y);
        const float2 e0 = __ffma2_rn(a1[j], shi[j], nq0);          // a1*s_hi - q0, exact
        const float2 m0 = __ffma2_rn(a0[j], chi[j], nq0);          // a0*c_hi - q0
        float2 l0 = __ffma2_rn(a0[j], clo[j], make_float2(-e0.x, -e0.y));
        l0 = __ffma2_rn(a1[j], make_float2(-slo[j].x, -slo[j].y), l0);
        y0[j] = __fmul2_rn(__fadd2_rn(m0, l0), rr);
        const float2 q1 = __fmul2_rn(a0[j], shi[j]);
        const float2 e1 = __ffma2_rn(a0[j], shi[j], make_float2(-q1.x, -q1.y));  // a0*s_hi - q1, exact
        const float2 m1 = __ffma2_rn(a1[j], chi[j], q1);           // a1*c_hi + q1
        float2 l1 = __ffma2_rn(a1[j], clo[j], e1);
        l1 = __ffma2_rn(a0[j], slo[j], l1);
        y1[j] = __fmul2_rn(__fadd2_rn(m1, l1), rr);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        y0[j] = __fmul2_rn(a0[j], rr);
        y1[j] = __fmul2_rn(a1[j], rr);
      }
    }
    if (live && store_in_bounds(token < p.n_tokens && h < n_heads && chunk * 8 + 8 <= D)) {
      // element 2i is the first of pair i: pair 2j + t sits in component t of couple j
      uint4 o;
      o.x = ptx::pack_bf16x2(y0[0].x, y1[0].x);
      o.y = ptx::pack_bf16x2(y0[0].y, y1[0].y);
      o.z = ptx::pack_bf16x2(y0[1].x, y1[1].x);
      o.w = ptx::pack_bf16x2(y0[1].y, y1[1].y);
      *reinterpret_cast<uint4*>(out) = o;
    }
    // Refill this slot (its value is consumed above) with the pass kPrologueDepth ahead; an
    // empty group keeps the group count in step at the tail.
    if (pass + kPrologueDepth < n_pass && h + kPrologueDepth * kHeadsPerPass < n_heads)
      cp_async16(&ring[warp][slot][lane], refill);
    cp_async_commit();
  }
}

}  // namespace h3
