// attention.cuh -- non-causal flash attention forward on sm_100a tensor cores.
//
// Computes O = softmax(Q K^T * scale) V per (sequence, head) over a packed
// token sequence, the dominant cost of the MiniMax-H3 DiT block ("Buyer
// Questions: Current Evidence Status", Q4 current answer: attention is the
// largest share of the profiled block; "Open-H3-Regenerate-2K", forward table:
// dense attention on one B200).  Ragged batches follow "H3 Runtime Current
// State" (ragged sequence parallelism): each cu_seqlens segment attends only to
// itself.
//
// One CTA per SM (640 threads = five warpgroups) owns two 128-row query tiles
// Q0, Q1 of one (sequence, head):
//   * warp 16 (one lane) -- TMA producer: Q0/Q1 once, then K_j and V_j tiles
//     (128 keys x d) into a ring of shared-memory slots, K and V alternating;
//   * warp 17 (one lane) -- tcgen05 MMA issuer: S_t = Q_t K_j^T into tensor
//     memory (fp32, 128 columns per tile); O_t += P_t V_j with P_t read from
//     tensor memory, where softmax wrote it over S_t.  Order per step j:
//     PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so the tensor core always holds the
//     other tile's work while one softmax group runs;
//   * warps 0-7 / 8-15 -- online softmax of Q0 / Q1.  Each query row (= one
//     tensor-memory lane) is shared by two threads in two warps of the same lane
//     quarter, one per 64-key half, so every scheduler runs two warps of the
//     active tile.  The halves trade their row maxima through shared memory
//     each step (an mbarrier orders it) and agree on one running max m (log2
//     units, may lag the true max by < 8 so that P <= 256 and O is rescaled
//     rarely); p = 2^(s*c - m) with c = scale*log2(e); P rounded to bf16 and
//     stored over S; l sums the rounded weights the PV product uses (they
//     normalise to exactly one), lx the unrounded ones (log-sum-exp);
//   * epilogue by the softmax warps: the halves add their row sums, each stores
//     its half of O / l as bf16; rows past the sequence end are not stored;
//     LSE = (m + log2 lx) * ln 2.
// Every barrier wait is bounded (common.cuh).
//
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 after.
// Shared memory: Q0, Q1 and kStages K/V slots, each 128 rows x d bf16 stored as
// d/64 blocks of 128 rows x 128 bytes with the 128-byte swizzle TMA writes and
// the MMA descriptors read (K-major for Q and K, MN-major for V).
#pragma once

#include <cuda.h>

#include <cstdint>

#include "common.cuh"

namespace h3 {

constexpr int kBM = 128;        // query rows per tile (tensor-memory lanes)
constexpr int kBN = 128;        // keys per K/V tile
constexpr int kQTiles = 2;      // query tiles per CTA
constexpr int kSoftmaxWarps = 16;
constexpr int kLoadWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kAttnThreads = 640;
// Registers: 640 threads launch at 96 per thread (five warps per scheduler x 96 <= 512);
// a softmax thread holds 64 scores, so every role fits without a setmaxnreg split.
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8

template <int D>
struct AttnTraits {
  static constexpr int kAtoms = D / 64;                      // 128-byte swizzle atoms along d
  static constexpr int kAtomBytes = kBM * 128;               // 128 rows x 128 bytes
  static constexpr int kTileBytes = kAtoms * kAtomBytes;     // one Q, K or V tile
  static constexpr int kStages = (D == 128) ? 4 : 8;         // K/V ring slots
  static constexpr int kTiles = kQTiles + kStages;
  // barriers: q, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], xch[2][4]
  static constexpr int kBarriers = 1 + 2 * kStages + 3 * kQTiles + kQTiles * 4;
  static constexpr int kXchBytes = 2 * kQTiles * 2 * kBM * 4;  // [parity][tile][half][row] fp32
  static constexpr int kSmemBytes =
      1024 /*alignment slack*/ + kTiles * kTileBytes + kXchBytes + 8 * kBarriers + 16;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(256 + kQTiles * D <= 512, "tensor memory budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct AttnParams {
  uint16_t* o;                // bf16 output
  int64_t o_batch, o_tok, o_head;
  float* lse;                 // may be null
  const int32_t* cu_seqlens;  // ragged only
  int32_t nseq;               // ragged only
  int32_t n_heads;
  int64_t seqlen;             // dense: tokens per sequence
  int64_t total;              // ragged: total tokens (LSE row stride per head)
  float scale_log2;           // softmax_scale * log2(e)
  LaunchCtl ctl;
};

// Bounded wait that ignores the launch-failed flag (used to drain copies in flight).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_test(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// 2^x for a pair of values x <= 8, on the FMA and integer pipes instead of the
// exponential unit.  x = n + f with n = rint(x) and f in [-1/2, 1/2]; 2^f by a
// degree-3 polynomial whose coefficients were fitted for this kernel by a Remez
// exchange on the relative error (max 7.5e-5 over [-1/2, 1/2], far below the 2^-8
// of the bf16 rounding that follows); 2^n is added to the exponent field.  x is
// clamped at -125 so the result stays a normal number (2^-125 where the exact
// value is smaller, e.g. masked keys: negligible next to a row sum >= 1).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer
  constexpr float kC0 = 0.9999280571937561f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.2426111251115799f, kC3 = 0.0551716685295105f;
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));         // n in the low mantissa bits
  const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));       // n as a float
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);        // x - n
  float2 q = __ffma2_rn(make_float2(kC3, kC3), f, make_float2(kC2, kC2));
  q = __ffma2_rn(q, f, make_float2(kC1, kC1));
  q = __ffma2_rn(q, f, make_float2(kC0, kC0));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// Every kEmuEvery-th pair of exponentials goes through exp2_poly2 (0 = none),
// moving part of the work from the exponential unit (16/clk/SM) to the FMA pipes.
#ifndef H3ATTN_EMU_EVERY
#define H3ATTN_EMU_EVERY 0
#endif
constexpr int kEmuEvery = H3ATTN_EMU_EVERY;

template <int D, bool kVarlen, bool kLse>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
  using T = AttnTraits<D>;
  constexpr int kS = T::kStages;
  extern __shared__ uint8_t smem_raw[];

  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t sQ = base;
  const uint32_t sKV = base + kQTiles * T::kTileBytes;
  float* const xch = reinterpret_cast<float*>(base_ptr + T::kTiles * T::kTileBytes);
  const uint32_t bars = base + T::kTiles * T::kTileBytes + T::kXchBytes;
  const uint32_t bar_q = bars;
  auto bar_kv_full = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_kv_empty = [&](int s) { return bars + 8u * (1 + kS + s); };
  auto bar_s_full = [&](int t) { return bars + 8u * (1 + 2 * kS + t); };
  auto bar_p_full = [&](int t) { return bars + 8u * (1 + 2 * kS + kQTiles + t); };
  auto bar_o_done = [&](int t) { return bars + 8u * (1 + 2 * kS + 2 * kQTiles + t); };
  auto bar_xch = [&](int t, int q) { return bars + 8u * (1 + 2 * kS + 3 * kQTiles + 4 * t + q); };
  volatile uint32_t* const slot_words = reinterpret_cast<volatile uint32_t*>(
      base_ptr + T::kTiles * T::kTileBytes + T::kXchBytes + 8 * T::kBarriers);
  // slot_words[0] = tensor-memory base, [1] = work valid, [2] = sequence, [3] = query-pair index

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LaunchCtl ctl = p.ctl;

  // ---- work decode (CTA-uniform, published through shared memory) ----------------
  if (threadIdx.x == 0) {
    uint32_t valid = launch_failed(ctl) ? 0u : 1u;
    uint32_t seq = 0, pair = blockIdx.x;
    if (kVarlen && valid) {
      valid = 0;
      uint32_t x = blockIdx.x;
      for (int s = 0; s < p.nseq; ++s) {
        const int32_t n = p.cu_seqlens[s + 1] - p.cu_seqlens[s];
        const uint32_t pairs = n > 0 ? static_cast<uint32_t>((n + kQTiles * kBM - 1) / (kQTiles * kBM)) : 0u;
        if (x < pairs) {
          valid = 1;
          seq = static_cast<uint32_t>(s);
          pair = x;
          break;
        }
        x -= pairs;
      }
    }
    slot_words[1] = valid;
    slot_words[2] = seq;
    slot_words[3] = pair;
  }
  __syncthreads();
  if (slot_words[1] == 0) return;  // CTA-uniform

  const int head = blockIdx.y;
  int batch = 0;
  int64_t seq_base = 0;  // first token of the sequence in the tensor's token dimension
  int64_t seq_len;
  if (kVarlen) {
    const int s = static_cast<int>(slot_words[2]);
    seq_base = p.cu_seqlens[s];
    seq_len = static_cast<int64_t>(p.cu_seqlens[s + 1]) - seq_base;
  } else {
    batch = blockIdx.z;
    seq_len = p.seqlen;
  }
  const int64_t q_row0 = static_cast<int64_t>(slot_words[3]) * (kQTiles * kBM);
  const int nkv = static_cast<int>((seq_len + kBN - 1) / kBN);
  const int kv_last_valid = static_cast<int>(seq_len - static_cast<int64_t>(nkv - 1) * kBN);

  // ---- setup: barriers and tensor memory --------------------------------------------
  if (warp == kLoadWarp && lane == 0) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < kS; ++s) {
      ptx::mbar_init(bar_kv_full(s), 1);
      ptx::mbar_init(bar_kv_empty(s), 1);
    }
    for (int t = 0; t < kQTiles; ++t) {
      ptx::mbar_init(bar_s_full(t), 1);
      ptx::mbar_init(bar_p_full(t), kSoftmaxWarps / kQTiles);
      ptx::mbar_init(bar_o_done(t), 1);
      for (int q = 0; q < 4; ++q) ptx::mbar_init(bar_xch(t, q), 64);
    }
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<uint32_t*>(slot_words)), T::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = slot_words[0];

  if (warp >= kSoftmaxWarps) {
    if (warp == kLoadWarp && lane == 0) {
      // ================================ TMA producer ================================
      bool ok = true;
      const int32_t y_seq = static_cast<int32_t>(seq_base);
      ptx::mbar_arrive_expect_tx(bar_q, kQTiles * T::kTileBytes);
      for (int t = 0; t < kQTiles; ++t)
        for (int a = 0; a < T::kAtoms; ++a)
          ptx::tma_load_4d(sQ + t * T::kTileBytes + a * T::kAtomBytes, &tm_q, bar_q, a * 64,
                           y_seq + static_cast<int32_t>(q_row0) + t * kBM, head, batch);
      uint32_t it = 0;
      for (int j = 0; j < nkv && ok; ++j) {
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int slot = static_cast<int>(it % kS);
          const uint32_t use = it / kS;
          if (use > 0 && !mbar_wait(bar_kv_empty(slot), (use - 1) & 1u, ctl)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bar_kv_full(slot), T::kTileBytes);
          const CUtensorMap* map = kv ? &tm_v : &tm_k;
          for (int a = 0; a < T::kAtoms; ++a)
            ptx::tma_load_4d(sKV + slot * T::kTileBytes + a * T::kAtomBytes, map, bar_kv_full(slot),
                             a * 64, y_seq + j * kBN, head, batch);
        }
      }
      if (ok) {
        // tail: the MMA warp's last releases must land before the CTA's smem is reused
        const uint32_t first = it > static_cast<uint32_t>(kS) ? it - kS : 0u;
        for (uint32_t u = first; u < it && ok; ++u)
          ok = mbar_wait(bar_kv_empty(static_cast<int>(u % kS)), (u / kS) & 1u, ctl);
      }
      if (!ok) {
        // failure: let the copies already issued land before the CTA releases its smem
        mbar_wait_for(bar_q, 0, 20000000ull);
        const uint32_t first = it > static_cast<uint32_t>(kS) ? it - kS : 0u;
        for (uint32_t u = first; u < it; ++u)
          mbar_wait_for(bar_kv_full(static_cast<int>(u % kS)), (u / kS) & 1u, 20000000ull);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ================================ MMA issuer ==================================
      constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBM, D, true);
      // Ring order of the producer: K_j is load 2j, V_j is load 2j+1.
      auto slot_of = [](uint32_t u) { return static_cast<int>(u % kS); };
      auto parity_of = [](uint32_t u) { return (u / kS) & 1u; };
      // The issuing lane shares its scheduler with busy softmax warps, so the issue
      // stream is kept minimal: fully unrolled, every descriptor a base low word plus
      // an immediate (descriptors differ only in the start address, bits 0-13).
      constexpr uint32_t kHi = ptx::sdesc_sw128_hi(1024);
      const uint32_t q_lo0 = ptx::sdesc_sw128_lo(sQ, 16);
      const uint32_t k_lo0 = ptx::sdesc_sw128_lo(sKV, 16);
      const uint32_t v_lo0 = ptx::sdesc_sw128_lo(sKV, T::kAtomBytes);
      constexpr uint32_t kTile16 = T::kTileBytes >> 4;
      auto issue_s = [&](int t, int ks) {
        const uint32_t qa = q_lo0 + t * kTile16, kb = k_lo0 + ks * kTile16;
        const uint32_t dS = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = ((kk >> 2) * T::kAtomBytes + (kk & 3) * 32) >> 4;
          ptx::mma_ss(dS, ptx::sdesc_make(qa + koff, kHi), ptx::sdesc_make(kb + koff, kHi), kIdescQK,
                      kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar_s_full(t));
      };
      // O_t += P_t V for the V tile in ring slot `vs`
      auto issue_pv = [&](int t, int vs, bool first) {
        const uint32_t vb = v_lo0 + vs * kTile16;
        const uint32_t dO = tmem + 256 + t * D, aP = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          ptx::mma_ts(dO, aP + kk * 8, ptx::sdesc_make(vb + ((kk * 16 * 128) >> 4), kHi), kIdescPV,
                      (!first || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(bar_o_done(t));
      };

      bool ok = mbar_wait(bar_q, 0, ctl) && mbar_wait(bar_kv_full(slot_of(0)), parity_of(0), ctl);
      if (ok) {
        ptx::tc_fence_after();
        for (int t = 0; t < kQTiles; ++t) issue_s(t, slot_of(0));
        ptx::mma_commit(bar_kv_empty(slot_of(0)));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const uint32_t uv = 2u * j + 1u, uk = 2u * j + 2u;
        const bool has_next = j + 1 < nkv;
        if (!mbar_wait(bar_kv_full(slot_of(uv)), parity_of(uv), ctl)) { ok = false; break; }
        for (int t = 0; t < kQTiles; ++t) {
          if (!mbar_wait(bar_p_full(t), static_cast<uint32_t>(j) & 1u, ctl)) { ok = false; break; }
          ptx::tc_fence_after();
          issue_pv(t, slot_of(uv), j == 0);
          if (t == kQTiles - 1) ptx::mma_commit(bar_kv_empty(slot_of(uv)));
          if (has_next) {
            // K_{j+1} is only needed here, after PV_t(j) has been issued
            if (t == 0 && !mbar_wait(bar_kv_full(slot_of(uk)), parity_of(uk), ctl)) { ok = false; break; }
            issue_s(t, slot_of(uk));
          }
        }
        if (!ok) break;
        if (has_next) ptx::mma_commit(bar_kv_empty(slot_of(uk)));
      }
    }
  } else {
    // ============================ softmax + epilogue ==============================
    const int t = warp >> 3;            // query tile
    const int half = (warp >> 2) & 1;   // which 64 keys of each row this thread owns
    const int quarter = warp & 3;       // tensor-memory lane quarter of this warp
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;                         // S / P columns
    const uint32_t tO = tmem + lane_off + 256 + t * D + half * (D / 2);    // this half of O
    const uint32_t xbar = bar_xch(t, quarter);
    constexpr int kParityStride = kQTiles * 2 * kBM;  // floats per exchange buffer
    float* const xmine = xch + ((t * 2 + half) * kBM + row_in_tile);
    float* const xpeer = xch + ((t * 2 + (half ^ 1)) * kBM + row_in_tile);
    const float c = p.scale_log2;
    float m = -INFINITY;  // running max of s*c (log2 units), possibly stale by < 8
    float l = 0.0f;       // this half's running sum of bf16(2^(s*c - m)): normalises O
    float lx = 0.0f;      // this half's running sum of 2^(s*c - m) in fp32: the log-sum-exp
    bool ok = true;
    uint32_t xphase = 0;  // phases completed on this row pair's exchange barrier

    for (int j = 0; j < nkv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(t), static_cast<uint32_t>(j) & 1u, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t sr[2][32];
      ptx::tmem_ld32(tS + half * 64, sr[0]);
      ptx::tmem_ld32(tS + half * 64 + 32, sr[1]);
      ptx::tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int i = 0; i < 32; ++i) s[q * 32 + i] = __uint_as_float(sr[q][i]);
      if (j == nkv - 1 && kv_last_valid < kBN) {
        const int lim = kv_last_valid - half * 64;  // keys of this half that exist
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= lim) s[i] = -INFINITY;
      }
      // this half's row max: four independent chains of three-input maxima
      float ma = fmaxf(s[0], s[1]), mb = fmaxf(s[2], s[3]);
      float mc = fmaxf(s[4], s[5]), md = fmaxf(s[6], s[7]);
#pragma unroll
      for (int i = 8; i < 64; i += 8) {
        ma = ptx::max3(ma, s[i], s[i + 1]);
        mb = ptx::max3(mb, s[i + 2], s[i + 3]);
        mc = ptx::max3(mc, s[i + 4], s[i + 5]);
        md = ptx::max3(md, s[i + 6], s[i + 7]);
      }
      // trade maxima with the other half of the row (buffers alternate by step parity)
      const int par = (j & 1) * kParityStride;
      xmine[par] = ptx::max3(ma, mb, fmaxf(mc, md));
      ptx::mbar_arrive(xbar);
      ok = __all_sync(0xffffffffu, mbar_wait(xbar, xphase & 1u, ctl));
      ++xphase;
      if (!ok) break;
      const float mx = fmaxf(xmine[par], xpeer[par]);
      const float cand = mx * c;
      const bool grow = cand > m + kRescaleThreshold;  // identical in both halves
      const float alpha = grow ? ptx::ex2_approx(m - cand) : 1.0f;
      if (grow) m = cand;
      l *= alpha;
      if (kLse) lx *= alpha;
      // P = 2^(s*c - m), rounded to bf16, written over S (this half: 32 packed columns)
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
      float2 acc[2], accx[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) acc[k] = accx[k] = make_float2(0.0f, 0.0f);
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), c2, nm2);
        float2 pe;
        if (kEmuEvery > 0 && (i % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1) {
          pe = exp2_poly2(x);
        } else {
          pe = make_float2(ptx::ex2_approx(x.x), ptx::ex2_approx(x.y));
        }
        pk[i] = ptx::pack_bf16x2(pe.x, pe.y);
        acc[i & 1] = __fadd2_rn(acc[i & 1], make_float2(__uint_as_float(pk[i] << 16),
                                                        __uint_as_float(pk[i] & 0xFFFF0000u)));
        if (kLse) accx[i & 1] = __fadd2_rn(accx[i & 1], pe);
      }
      ptx::tmem_st32(tS + half * 32, pk);
      {
        const float2 a = __fadd2_rn(acc[0], acc[1]);
        l += a.x + a.y;
        if (kLse) {
          const float2 b = __fadd2_rn(accx[0], accx[1]);
          lx += b.x + b.y;
        }
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O_t(j-1) is final once S_t(j) has landed (the tensor core runs in issue
        // order); the explicit wait keeps that visible.  Rescale this half in place.
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done(t), static_cast<uint32_t>(j - 1) & 1u, ctl));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
          uint32_t orr[32];
          ptx::tmem_ld32(tO + q * 32, orr);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          ptx::tmem_st32(tO + q * 32, orr);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_p_full(t));  // one arrival per warp
    }

    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done(t), static_cast<uint32_t>(nkv - 1) & 1u, ctl));
    }
    if (ok) {
      // the two halves add their row sums (the buffer the last step did not use)
      const int par = (nkv & 1) * kParityStride;
      xmine[par] = l;
      ptx::mbar_arrive(xbar);
      ok = __all_sync(0xffffffffu, mbar_wait(xbar, xphase & 1u, ctl));
      ++xphase;
    }
    if (ok) {
      const int par = (nkv & 1) * kParityStride;
      const float l_row = xmine[par] + xpeer[par];
      ptx::tc_fence_after();
      const int64_t row = q_row0 + t * kBM + row_in_tile;  // within the sequence
      const bool valid = row < seq_len;
      const float inv_l = 1.0f / l_row;
      uint16_t* orow = p.o + static_cast<int64_t>(batch) * p.o_batch + (seq_base + row) * p.o_tok +
                       static_cast<int64_t>(head) * p.o_head + half * (D / 2);
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        uint32_t orr[32];
        ptx::tmem_ld32(tO + q * 32, orr);
        ptx::tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = ptx::pack_bf16x2(__uint_as_float(orr[2 * i]) * inv_l, __uint_as_float(orr[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (kLse) {
        // a second round for the unrounded sums, in the other buffer (whose last
        // reader, the peer's final step, finished before the round above)
        const int par2 = ((nkv + 1) & 1) * kParityStride;
        xmine[par2] = lx;
        ptx::mbar_arrive(xbar);
        ok = __all_sync(0xffffffffu, mbar_wait(xbar, xphase & 1u, ctl));
        ++xphase;
        if (ok && half == 0 && valid) {
          const float lx_row = xmine[par2] + xpeer[par2];
          const float v = (m + log2f(lx_row)) * 0.69314718055994530942f;
          if (kVarlen) {
            p.lse[static_cast<int64_t>(head) * p.total + seq_base + row] = v;
          } else {
            p.lse[(static_cast<int64_t>(batch) * p.n_heads + head) * p.seqlen + row] = v;
          }
        }
      }
    }
  }

  // ---- teardown: every thread arrives here, then the allocating warp frees TMEM ----
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, T::kTmemCols);
  }
}

}  // namespace h3
