// qkv.cuh -- the Q/K/V projection of the block with the Q/K RMSNorm + RoPE fused
// into its epilogue.
//
// "H3 Runtime Current State" (Owned Performance Kernels) lists "fused Q/K
// RMSNorm, RoPE, and layout work" as missing, and "Buyer Questions: Current
// Evidence Status" (block composition) books the projection, then norm/RoPE,
// ahead of attention, with the strided NHD layout of the projection output read
// in place.  Here the norm, the rotation and the NHD layout are the epilogue of
// the projection GEMM itself: the fp32 accumulator of a (128 tokens x 256
// features) tile is normalised per head, rotated, rounded once to bf16 and
// written straight into Q', K', V; no intermediate tensor is stored or read.
//
//   feature f = sum_c X[n][c] * W[f][c] (+ bias[f]), f in [0, 3*H*d):
//   [0, H*d) Q, [H*d, 2*H*d) K, [2*H*d, 3*H*d) V, head = (f mod H*d) / d.
//
// Persistent kernel, one CTA per SM (320 threads):
//   * warp 0 (one lane) -- TMA producer: X tile [128 tokens x 64] and W tile
//     [256 features x 64] per K step into a 4-slot ring (48 KB a slot, 128-byte
//     swizzle; rows past the token count read as zero);
//   * warp 1 (one lane) -- tcgen05 issuer: D[128 x 256] += X W^T, four
//     M128 N256 K16 MMAs per K step, into one of two tensor-memory accumulators
//     (2 x 256 columns) so the epilogue of one tile overlaps the next tile's
//     main loop;
//   * warps 2-9 -- epilogue: a warp owns 32 token rows (its tensor-memory lane
//     quarter) and 128 of the tile's 256 features; each thread one token row,
//     32 accumulator columns at a time (a first pass over a Q/K head forms the
//     sum of squares); results go through a per-warp 2 KB shared-memory block
//     (32 tokens x 32 features in the 64-byte swizzle), which the CTA-pair kernel
//     writes out with one bulk tensor store per block and the single-CTA kernel
//     with row-contiguous 16-byte stores (four lanes per row).  Q/K heads: RMS in fp32, x * (1/rms) * gamma, then RoPE
//     with the angle formed and reduced to [-pi, pi] in fp32 with error-free
//     products (frequency and 2 pi carried as float pairs) and cos/sin from the
//     fp32 intrinsic (the projection's fp32 accumulation error dominates here,
//     unlike in the standalone prologue whose input is exact); V: bias and
//     rounding only.
// Tiles are numbered feature-tile fastest, so the CTAs running at once share a
// few X row blocks and W stays resident in L2 (3*H*d x dim_in bf16 = 57 MB at
// H*d = dim_in = 3072).  Every barrier wait is bounded (common.cuh).
//
// qkv_fused_pair_kernel (below) is the same design on CTA pairs: 256-token tiles
// whose M256 MMAs span two SMs, each CTA staging half the operands; the host
// launches it unless the library is built with H3_QKV_PAIRS=0.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "common.cuh"
#include "prologue.cuh"

namespace h3 {

constexpr int kGemmBM = 128;      // tokens per tile (tensor-memory lanes)
constexpr int kGemmBN = 256;      // output features per tile
constexpr int kGemmBK = 64;       // K elements per stage (one 128-byte swizzle row)
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 320;
constexpr int kGemmEpiWarp0 = 2;  // warps 2..9: epilogue
constexpr int kGemmEpiWarps = 8;

// Rotary frequencies as float pairs (hi + lo = the fp64 value to ~2^-48): the
// epilogue forms p * f and reduces it modulo 2 pi in fp32 arithmetic with
// error-free products, without fp64 (which is slow on this part).
struct RopeTablesF {
  float hi3[kRopeMaxPairs], lo3[kRopeMaxPairs];  // 3D layout, pair p inside its section
  float hi1[kRopeMaxPairs], lo1[kRopeMaxPairs];  // 1D layout
  uint8_t axis3[kRopeMaxPairs];                  // 0 = t, 1 = h, 2 = w
};

struct QkvParams {
  uint16_t* out[3];           // Q', K', V (bf16)
  int64_t out_tok[3];         // element strides
  int64_t out_head[3];
  const uint16_t* bias;       // [3*H*d] or null
  const uint16_t* gamma[2];   // [d] or null (Q, K)
  const int32_t* pos;         // [n_tokens][3] or null
  const uint8_t* kind;        // [n_tokens]
  RopeTablesF rope;
  int64_t n_tokens;
  int32_t dim_in;
  int32_t n_heads;
  float eps;
  int32_t m_tiles, n_tiles;
  LaunchCtl ctl;
};

struct QkvTraits {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;   // 16 KB
  static constexpr int kBBytes = kGemmBN * kGemmBK * 2;   // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2], drain; the area is
  // padded to 16 bytes so the staging blocks after it stay 16-byte aligned
  static constexpr int kBarriers = 2 * kGemmStages + 5;
  static constexpr int kBarrierBytes = (8 * kBarriers + 15) / 16 * 16;
  // per epilogue warp: a 32-row x 32-column bf16 staging block (2 KB) that turns
  // its thread-per-row results into row-contiguous global stores
  static constexpr int kStageOutBytes = 32 * 32 * 2;
  static constexpr int kSmemBytes =
      1024 + kGemmStages * kStageBytes + kBarrierBytes + 16 + kGemmEpiWarps * kStageOutBytes;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert((kGemmStages * kStageBytes + kBarrierBytes + 16) % 16 == 0, "staging blocks 16-byte aligned");
};

// The CTA-pair variant: a cluster of two CTAs computes a 256-token x 256-feature
// tile with M256 N256 MMAs issued by rank 0.  Each CTA stages per K step only
// its own 128 tokens of X and 128 of the tile's 256 W rows (32 KB, against
// 48 KB for a 128 x 256 tile alone), so shared-memory and L2 traffic per MMA
// drop by a third and six stages fit.  Its epilogue is the single-CTA one, on
// the 128 x 256 accumulator that each CTA holds.
struct QkvPairTraits {
  static constexpr int kStages = 6;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;        // 16 KB: this CTA's 128 tokens
  static constexpr int kBBytes = (kGemmBN / 2) * kGemmBK * 2;  // 16 KB: this CTA's 128 W rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarriers = 2 * kStages + 5;
  static constexpr int kBarrierBytes = (8 * kBarriers + 15) / 16 * 16;
  static constexpr int kStageOutBytes = QkvTraits::kStageOutBytes;
  // layout: stages | output staging blocks (1024-byte aligned: the 64-byte swizzle
  // of the bulk tensor stores is taken from address bits) | barriers | slot words
  static constexpr int kSmemBytes =
      1024 + kStages * kStageBytes + kGemmEpiWarps * kStageOutBytes + kBarrierBytes + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert((kStages * kStageBytes) % 1024 == 0, "staging blocks 1024-byte aligned");
};
constexpr int kGemmPairBM = 2 * kGemmBM;  // tokens per pair tile

// Epilogue of one accumulator tile for one warp: its 32 token rows (TMEM lane
// quarter `quarter`; tokens m_row0 + 32 * quarter + lane) and 128 of the tile's 256
// features (`half`), read from tensor memory at tacc.  Q/K: bias, RMS norm, gamma,
// RoPE; V: bias; all rounded once to bf16 and stored through the warp's staging
// block wstage.
template <int D, bool kBulkStore = false>
__device__ __forceinline__ void qkv_epilogue_tile(const QkvParams& p, int64_t m_row0, int nt, int quarter,
                                                  int half, int lane, uint32_t tacc, uint8_t* wstage,
                                                  const CUtensorMap* const* out_maps = nullptr) {
  const int hd = p.n_heads * D;
  const int row = quarter * 32 + lane;  // token row inside the tile
  const int f0 = nt * kGemmBN + half * 128;  // first feature of this warp's 128
  const int part = f0 / hd;                  // 0 Q, 1 K, 2 V
  const int64_t n = m_row0 + row;
  const bool valid = n < p.n_tokens;

  // cos/sin of this token's pairs (Q and K tiles with RoPE only)
  const bool rope = part < 2 && p.pos != nullptr && valid && p.kind[valid ? n : 0] != 0;
  const int kd = rope ? p.kind[n] : 0;
  int32_t pt0 = 0, pt1 = 0, pt2 = 0;
  if (rope) {
    pt0 = p.pos[3 * n];
    pt1 = p.pos[3 * n + 1];
    pt2 = p.pos[3 * n + 2];
  }
#pragma unroll 1
  for (int h0 = 0; h0 < 128; h0 += D) {      // the heads among this warp's 128 features
    const int head = (f0 + h0 - part * hd) / D;
    const uint4* const bias4 = p.bias ? reinterpret_cast<const uint4*>(p.bias + f0 + h0) : nullptr;
    const bool norm = part < 2 && p.gamma[part] != nullptr;
    // bias of 32 columns starting at c, added to v; 16-byte loads at the same
    // addresses in every thread (served once per warp)
    auto add_bias = [&](int c, float* v) {
      if (bias4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 bv = __ldg(bias4 + c / 8 + q);
          const uint32_t w4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[8 * q + 2 * i] += __uint_as_float(w4[i] << 16);
            v[8 * q + 2 * i + 1] += __uint_as_float(w4[i] & 0xFFFF0000u);
          }
        }
      }
    };
    // pass 1 (Q, K): the row's sum of squares -- all of the head's columns in
    // flight at once, one wait; they are read again below
    float rinv = 1.0f;
    if (norm) {
      uint32_t ra[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(tacc + h0 + 32 * c, ra[c]);
      ptx::tmem_wait_ld();
      float ss = 0.0f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(ra[c][i]);
        add_bias(32 * c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      rinv = rsqrtf(ss / static_cast<float>(D) + p.eps);
    }
    // pass 2: scale, rotate, round, store -- 64 columns per wait, 32 at a time
#pragma unroll
    for (int c2 = 0; c2 < D; c2 += 64) {
      uint32_t rb[2][32];
      ptx::tmem_ld32(tacc + h0 + c2, rb[0]);
      ptx::tmem_ld32(tacc + h0 + c2 + 32, rb[1]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int c = c2 + 32 * hh;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rb[hh][i]);
        add_bias(c, v);
        if (norm) {
          const uint4* g = reinterpret_cast<const uint4*>(p.gamma[part]) + c / 8;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 gv = __ldg(g + q);
            const uint32_t w4[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[8 * q + 2 * i] = (v[8 * q + 2 * i] * rinv) * __uint_as_float(w4[i] << 16);
              v[8 * q + 2 * i + 1] = (v[8 * q + 2 * i + 1] * rinv) * __uint_as_float(w4[i] & 0xFFFF0000u);
            }
          }
        }
        if (rope) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int pr = c / 2 + i;  // rotation pair of columns (2 pr, 2 pr + 1)
            float pf, fh, fl;          // position (exact) and frequency hi + lo
            if (kd == 1) {
              const int ax = p.rope.axis3[pr];
              pf = static_cast<float>(ax == 0 ? pt0 : ax == 1 ? pt1 : pt2);
              fh = p.rope.hi3[pr];
              fl = p.rope.lo3[pr];
            } else {
              pf = static_cast<float>(pt0);
              fh = p.rope.hi1[pr];
              fl = p.rope.lo1[pr];
            }
            // angle = pf * (fh + fl) as prod + tail (prod + e exact), reduced modulo
            // 2 pi (2 pi as hi + lo): |error| ~ 2^-24 pi + |angle| 2^-46 before cos/sin
            const float prod = pf * fh;
            const float tail = fmaf(pf, fh, -prod) + pf * fl;
            const float turns = rintf(prod * 0.159154943091895336f);
            float red = fmaf(-turns, 6.28318548202514648f, prod);   // 2 pi rounded to float
            red = fmaf(-turns, -1.74845553e-7f, red) + tail;           // 2 pi = that + this
            float sn, cs;
            __sincosf(red, &sn, &cs);
            const float a0 = v[2 * i], a1 = v[2 * i + 1];
            v[2 * i] = fmaf(a0, cs, -a1 * sn);
            v[2 * i + 1] = fmaf(a0, sn, a1 * cs);
          }
        }
        // stage this thread's 32 columns (four 16-byte pieces of its row) in the
        // warp's block, pieces swizzled by row so that the writes and the
        // row-wise reads below are free of bank conflicts
        if (kBulkStore) {  // the block's previous bulk store must have read it
          if (lane == 0) ptx::bulk_wait_read_all();
          __syncwarp();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int sw = q ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(wstage + lane * 64 + sw * 16) =
              make_uint4(ptx::pack_bf16x2(v[8 * q], v[8 * q + 1]), ptx::pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                         ptx::pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), ptx::pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        }
        if (kBulkStore) {
          // one bulk tensor store of the 32 x 32 block (the swizzle above is the
          // tensor map's 64-byte swizzle); rows past the last token are clipped
          ptx::fence_proxy_async_smem();
          __syncwarp();
          const int64_t tok0 = m_row0 + quarter * 32;
          if (lane == 0 && tok0 < p.n_tokens && store_in_bounds(head < p.n_heads && c + 32 <= D)) {
            ptx::tma_store_3d(out_maps[part], ptx::smem_u32(wstage), c, head, static_cast<int32_t>(tok0));
            ptx::bulk_commit_group();
          }
          continue;
        }
        __syncwarp();
        // row-contiguous stores: lanes 4r..4r+3 write the 64 bytes of one row
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int srow = rr * 8 + (lane >> 2), piece = lane & 3;
          const int64_t tok = m_row0 + quarter * 32 + srow;
          const uint4 val =
              *reinterpret_cast<const uint4*>(wstage + srow * 64 + (piece ^ ((srow >> 1) & 3)) * 16);
          if (tok < p.n_tokens && store_in_bounds(head < p.n_heads && c + 32 <= D && part < 3)) {
            uint16_t* const drow = p.out[part] + tok * p.out_tok[part] +
                                   static_cast<int64_t>(head) * p.out_head[part] + c;
            *reinterpret_cast<uint4*>(drow + piece * 8) = val;
          }
        }
        __syncwarp();  // the block is reused by the next 32 columns
      }
    }
  }
}

// rows past n_tokens are never written; every thread reaches the final barrier
template <int D>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qkv_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ QkvParams p) {
  using T = QkvTraits;
  constexpr int kS = kGemmStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t bars = base + kS * T::kStageBytes;
  auto bar_full = [&](int s) { return bars + 8u * s; };
  auto bar_empty = [&](int s) { return bars + 8u * (kS + s); };
  auto bar_acc_full = [&](int b) { return bars + 8u * (2 * kS + b); };
  auto bar_acc_empty = [&](int b) { return bars + 8u * (2 * kS + 2 + b); };
  const uint32_t bar_drain = bars + 8u * (2 * kS + 4);  // MMA lane's exit after a failure
  volatile uint32_t* const slot = reinterpret_cast<volatile uint32_t*>(base_ptr + kS * T::kStageBytes + T::kBarrierBytes);
  uint8_t* const stage_out = base_ptr + kS * T::kStageBytes + T::kBarrierBytes + 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LaunchCtl ctl = p.ctl;
  const int n_total = p.m_tiles * p.n_tiles;
  const int k_steps = p.dim_in / kGemmBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kS; ++s) {
      ptx::mbar_init(bar_full(s), 1);
      ptx::mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar_acc_full(b), 1);
      ptx::mbar_init(bar_acc_empty(b), kGemmEpiWarps);
    }
    ptx::mbar_init(bar_drain, 1);
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tm_x);
    ptx::tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<uint32_t*>(slot)), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = slot[0];

  if (warp == 0) {
    if (lane == 0) {
      // ================================ TMA producer ================================
      bool ok = true;
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < n_total && ok; tile += gridDim.x) {
        const int m = tile / p.n_tiles, nt = tile % p.n_tiles;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = static_cast<int>(it % kS);
          const uint32_t use = it / kS;
          if (use > 0 && !mbar_wait(bar_empty(s), (use - 1) & 1u, ctl)) {
            ok = false;
            break;
          }
          const uint32_t dst = base + s * T::kStageBytes;
          ptx::mbar_arrive_expect_tx(bar_full(s), T::kStageBytes);
          ptx::tma_load_4d(dst, &tm_x, bar_full(s), ks * kGemmBK, m * kGemmBM, 0, 0);
          ptx::tma_load_4d(dst + T::kABytes, &tm_w, bar_full(s), ks * kGemmBK, nt * kGemmBN, 0, 0);
        }
      }
      // drain: the last copies must land before the CTA's shared memory is released
      const uint32_t first = it > static_cast<uint32_t>(kS) ? it - kS : 0u;
      for (uint32_t u = first; u < it; ++u) {
        const uint64_t t0 = ptx::globaltimer_ns();
        while (!ptx::mbar_test(bar_full(static_cast<int>(u % kS)), (u / kS) & 1u)) {
          if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================ MMA issuer ==================================
      constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kGemmBM, kGemmBN, false);
      constexpr uint32_t kHi = ptx::sdesc_sw128_hi(1024);
      bool ok = true;
      uint32_t it = 0;
      int k = 0;  // this CTA's tile counter
      for (int tile = blockIdx.x; tile < n_total && ok; tile += gridDim.x, ++k) {
        const int buf = k & 1;
        if (k >= 2 && !mbar_wait(bar_acc_empty(buf), static_cast<uint32_t>((k >> 1) - 1) & 1u, ctl)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t acc = tmem + buf * kGemmBN;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = static_cast<int>(it % kS);
          if (!mbar_wait(bar_full(s), (it / kS) & 1u, ctl)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_lo = ptx::sdesc_sw128_lo(base + s * T::kStageBytes, 16);
          const uint32_t b_lo = ptx::sdesc_sw128_lo(base + s * T::kStageBytes + T::kABytes, 16);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
            ptx::mma_ss(acc, ptx::sdesc_make(a_lo + kk * 2, kHi), ptx::sdesc_make(b_lo + kk * 2, kHi), kIdesc,
                        (ks > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(bar_empty(s));
        }
        if (ok) ptx::mma_commit(bar_acc_full(buf));
      }
      if (!ok) {
        // failure: every MMA already issued must finish writing tensor memory
        // before the teardown frees it
        ptx::mma_commit(bar_drain);
        mbar_wait_for(bar_drain, 0, kDrainLimitNs);
      }
    }
  } else {
    // ================================= epilogue ===================================
    const int ew = warp - kGemmEpiWarp0;   // 0..7
    const int quarter = warp & 3;          // tensor-memory lane quarter of this warp
    const int half = ew >> 2;              // which 128 of the tile's 256 features
    uint8_t* const wstage = stage_out + ew * T::kStageOutBytes;
    bool ok = true;
    int k = 0;
    for (int tile = blockIdx.x; tile < n_total; tile += gridDim.x, ++k) {
      const int buf = k & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full(buf), static_cast<uint32_t>(k >> 1) & 1u, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      const int m = tile / p.n_tiles, nt = tile % p.n_tiles;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kGemmBN + half * 128;
      qkv_epilogue_tile<D>(p, static_cast<int64_t>(m) * kGemmBM, nt, quarter, half, lane, tacc, wstage);
      // the accumulator is read: the tensor core may reuse it
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_acc_empty(buf));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// CTA-pair kernel (cluster of two): tiles of 256 tokens x 256 features, numbered
// as in the single-CTA kernel with p.m_tiles counting 256-token tiles.  Rank r of
// the pair loads tokens 128 r.. of the tile and W rows 128 r.. of its 256 and
// writes the outputs of its 128 tokens.  Barriers: full[s] lives in rank 0 and
// counts both CTAs' bytes; empty[s] and acc_full[b] exist in both CTAs and are
// signalled by rank 0's commits to both; acc_empty[b] lives in rank 0 and takes
// an arrival from each of the 16 epilogue warps of the pair.  Every wait is
// bounded and every thread of both CTAs reaches the final cluster barrier.
template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    qkv_fused_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                          const __grid_constant__ CUtensorMap tm_oq, const __grid_constant__ CUtensorMap tm_ok,
                          const __grid_constant__ CUtensorMap tm_ov, const __grid_constant__ QkvParams p) {
  using T = QkvPairTraits;
  constexpr int kS = T::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t bars = base + kS * T::kStageBytes + kGemmEpiWarps * T::kStageOutBytes;
  auto bar_full = [&](int s) { return bars + 8u * s; };
  auto bar_empty = [&](int s) { return bars + 8u * (kS + s); };
  auto bar_acc_full = [&](int b) { return bars + 8u * (2 * kS + b); };
  auto bar_acc_empty = [&](int b) { return bars + 8u * (2 * kS + 2 + b); };
  const uint32_t bar_drain = bars + 8u * (2 * kS + 4);  // MMA lane's exit after a failure
  uint8_t* const stage_out = base_ptr + kS * T::kStageBytes;
  volatile uint32_t* const slot = reinterpret_cast<volatile uint32_t*>(
      base_ptr + kS * T::kStageBytes + kGemmEpiWarps * T::kStageOutBytes + T::kBarrierBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);
  const LaunchCtl ctl = p.ctl;
  const int n_total = p.m_tiles * p.n_tiles;
  const int k_steps = p.dim_in / kGemmBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kS; ++s) {
      ptx::mbar_init(bar_full(s), 1);
      ptx::mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar_acc_full(b), 1);
      ptx::mbar_init(bar_acc_empty(b), 2 * kGemmEpiWarps);
    }
    ptx::mbar_init(bar_drain, 1);
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tm_x);
    ptx::tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(const_cast<uint32_t*>(slot)), 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  ptx::tc_fence_after();
  const uint32_t tmem = slot[0];

  if (warp == 0) {
    if (lane == 0) {
      // ================================ TMA producer ================================
      bool ok = true;
      uint32_t it = 0;
      for (int tile = pair; tile < n_total && ok; tile += n_pairs) {
        const int m = tile / p.n_tiles, nt = tile % p.n_tiles;
        const int32_t row_x = m * kGemmPairBM + static_cast<int32_t>(rank) * kGemmBM;
        const int32_t row_w = nt * kGemmBN + static_cast<int32_t>(rank) * (kGemmBN / 2);
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = static_cast<int>(it % kS);
          const uint32_t use = it / kS;
          if (use > 0 && !mbar_wait(bar_empty(s), (use - 1) & 1u, ctl)) {
            ok = false;
            break;
          }
          const uint32_t dst = base + s * T::kStageBytes;
          const uint32_t full0 = ptx::map_shared_rank(bar_full(s), 0);
          if (rank == 0) ptx::mbar_arrive_expect_tx(bar_full(s), 2 * T::kStageBytes);
          ptx::tma_load_4d_pair(dst, &tm_x, full0, ks * kGemmBK, row_x, 0, 0);
          ptx::tma_load_4d_pair(dst + T::kABytes, &tm_w, full0, ks * kGemmBK, row_w, 0, 0);
        }
      }
      // tail: every stage released by rank 0's MMAs, so no commit is still on its
      // way to this CTA's barriers when it exits
      const uint32_t first = it > static_cast<uint32_t>(kS) ? it - kS : 0u;
      for (uint32_t u = first; u < it && ok; ++u)
        ok = mbar_wait(bar_empty(static_cast<int>(u % kS)), (u / kS) & 1u, ctl);
      // drain after a failure (rank 0 holds the barriers that count both CTAs'
      // copies): the last copies must land before either CTA's shared memory is
      // released
      if (rank == 0 && !ok) {
        for (uint32_t u = first; u < it; ++u) {
          const uint64_t t0 = ptx::globaltimer_ns();
          while (!ptx::mbar_test(bar_full(static_cast<int>(u % kS)), (u / kS) & 1u)) {
            if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) break;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ========================= MMA issuer (rank 0 only) ===========================
      constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kGemmPairBM, kGemmBN, false);
      constexpr uint32_t kHi = ptx::sdesc_sw128_hi(1024);
      constexpr uint16_t kBoth = 0x3;
      bool ok = true;
      uint32_t it = 0;
      int k = 0;  // this pair's tile counter
      for (int tile = pair; tile < n_total && ok; tile += n_pairs, ++k) {
        const int buf = k & 1;
        if (k >= 2 && !mbar_wait(bar_acc_empty(buf), static_cast<uint32_t>((k >> 1) - 1) & 1u, ctl)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t acc = tmem + buf * kGemmBN;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = static_cast<int>(it % kS);
          if (!mbar_wait(bar_full(s), (it / kS) & 1u, ctl)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_lo = ptx::sdesc_sw128_lo(base + s * T::kStageBytes, 16);
          const uint32_t b_lo = ptx::sdesc_sw128_lo(base + s * T::kStageBytes + T::kABytes, 16);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
            ptx::mma_ss_pair(acc, ptx::sdesc_make(a_lo + kk * 2, kHi), ptx::sdesc_make(b_lo + kk * 2, kHi), kIdesc,
                             (ks > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit_pair(bar_empty(s), kBoth);
        }
        if (ok) ptx::mma_commit_pair(bar_acc_full(buf), kBoth);
      }
      // tail: both accumulators released by the 16 epilogue warps, so no peer
      // arrival is still on its way to this CTA when it exits
      for (int j = k >= 2 ? k - 2 : 0; j < k && ok; ++j)
        ok = mbar_wait(bar_acc_empty(j & 1), static_cast<uint32_t>(j >> 1) & 1u, ctl);
      if (!ok) {
        // failure: every pair MMA already issued must finish writing both CTAs'
        // tensor memory before the teardown frees it (arrives on rank 0 only)
        ptx::mma_commit_pair(bar_drain, 0x1);
        mbar_wait_for(bar_drain, 0, kDrainLimitNs);
      }
    }
  } else {
    // ================================= epilogue ===================================
    const int ew = warp - kGemmEpiWarp0;   // 0..7
    const int quarter = warp & 3;          // tensor-memory lane quarter of this warp
    const int half = ew >> 2;              // which 128 of the tile's 256 features
    uint8_t* const wstage = stage_out + ew * T::kStageOutBytes;
    bool ok = true;
    int k = 0;
    for (int tile = pair; tile < n_total; tile += n_pairs, ++k) {
      const int buf = k & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full(buf), static_cast<uint32_t>(k >> 1) & 1u, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      const int m = tile / p.n_tiles, nt = tile % p.n_tiles;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kGemmBN + half * 128;
      const CUtensorMap* const maps[3] = {&tm_oq, &tm_ok, &tm_ov};
      qkv_epilogue_tile<D, true>(p, static_cast<int64_t>(m) * kGemmPairBM + static_cast<int64_t>(rank) * kGemmBM,
                                 nt, quarter, half, lane, tacc, wstage, maps);
      // the accumulator is read: rank 0's tensor core may reuse it
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::map_shared_rank(bar_acc_empty(buf), 0));
    }
  }

  if (warp >= kGemmEpiWarp0 && lane == 0) ptx::bulk_wait_all();  // this warp's output stores are done
  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();  // no CTA leaves while its peer may still signal or read it
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace h3
