// merge.cuh -- combination of two partial attention results by log-sum-exp.
//
// A key-split schedule of the sequence-parallel attention ("H3 Runtime Current
// State": ragged Ulysses sequence parallelism, sequence-sharded block execution)
// computes, for the same query rows, attention over disjoint blocks of keys;
// each block gives O_p (the block's softmax-weighted mean of values) and LSE_p
// (the log of the block's total weight).  Their combination is the attention
// over all keys:
//   L = log(exp(LSE_a) + exp(LSE_b)) = M + log(exp(LSE_a - M) + exp(LSE_b - M)),
//   O = exp(LSE_a - L) O_a + exp(LSE_b - L) O_b,          M = max(LSE_a, LSE_b).
// An empty block has LSE = -inf and weight 0; both empty gives O = 0, L = -inf.
//
// HBM-bound: per (token, head) row it reads two rows of d bf16 and two fp32
// LSE values and writes one row and one LSE.  A block owns 64 tokens of one
// (batch, head): 64 threads form the weights from coalesced LSE reads, then
// every warp streams whole rows with 16-byte loads and stores (a d = 128 row is
// 16 lanes x 16 bytes).  In place is allowed (O = O_a, LSE = LSE_a): every
// element is read and written by the same thread.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace h3 {

constexpr int kMergeTokens = 64;   // tokens per block
constexpr int kMergeThreads = 256;

struct MergeParams {
  const uint16_t* oa;
  const uint16_t* ob;
  uint16_t* o;
  int64_t oa_batch, oa_tok, oa_head;  // element strides
  int64_t ob_batch, ob_tok, ob_head;
  int64_t o_batch, o_tok, o_head;
  const float* lse_a;  // [batch][n_heads][seqlen]
  const float* lse_b;
  float* lse;
  int64_t seqlen;
  int32_t n_heads;
};

template <int D>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ MergeParams p) {
  __shared__ float s_wa[kMergeTokens], s_wb[kMergeTokens];
  const int head = blockIdx.y, batch = blockIdx.z;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kMergeTokens;
  const int64_t lrow = (static_cast<int64_t>(batch) * p.n_heads + head) * p.seqlen;
  if (threadIdx.x < kMergeTokens) {
    const int64_t n = n0 + threadIdx.x;
    float wa = 0.0f, wb = 0.0f;
    if (n < p.seqlen) {
      const float la = p.lse_a[lrow + n], lb = p.lse_b[lrow + n];
      const float m = fmaxf(la, lb);
      float L = -INFINITY;
      if (m != -INFINITY) {
        const float ea = expf(la - m), eb = expf(lb - m);  // the larger one is exactly 1
        const float sum = ea + eb;
        L = m + logf(sum);
        wa = ea / sum;
        wb = eb / sum;
      }
      if (store_in_bounds(head < p.n_heads && batch < static_cast<int64_t>(gridDim.z))) p.lse[lrow + n] = L;
    }
    s_wa[threadIdx.x] = wa;
    s_wb[threadIdx.x] = wb;
  }
  __syncthreads();
  constexpr int kLanesPerRow = D / 8;            // 16-byte chunks of a row
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  constexpr int kRowsPerPass = (kMergeThreads / 32) * kRowsPerWarp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, chunk = lane % kLanesPerRow;
  for (int r = warp * kRowsPerWarp + sub; r < kMergeTokens; r += kRowsPerPass) {
    const int64_t n = n0 + r;
    if (n >= p.seqlen) break;
    const float wa = s_wa[r], wb = s_wb[r];
    const uint4 va = *reinterpret_cast<const uint4*>(p.oa + batch * p.oa_batch + n * p.oa_tok +
                                                     head * p.oa_head + chunk * 8);
    const uint4 vb = *reinterpret_cast<const uint4*>(p.ob + batch * p.ob_batch + n * p.ob_tok +
                                                     head * p.ob_head + chunk * 8);
    const uint32_t a[4] = {va.x, va.y, va.z, va.w}, b[4] = {vb.x, vb.y, vb.z, vb.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a_lo = __uint_as_float(a[i] << 16), a_hi = __uint_as_float(a[i] & 0xFFFF0000u);
      const float b_lo = __uint_as_float(b[i] << 16), b_hi = __uint_as_float(b[i] & 0xFFFF0000u);
      out[i] = ptx::pack_bf16x2(fmaf(wa, a_lo, wb * b_lo), fmaf(wa, a_hi, wb * b_hi));
    }
    if (store_in_bounds(n < p.seqlen && head < p.n_heads && batch < static_cast<int64_t>(gridDim.z) &&
                        chunk * 8 + 8 <= D))
      *reinterpret_cast<uint4*>(p.o + batch * p.o_batch + n * p.o_tok + head * p.o_head + chunk * 8) =
          make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace h3
