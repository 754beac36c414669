// attention.cuh -- non-causal flash attention forward on sm_100a tensor cores.
//
// Computes O = softmax(Q K^T * scale) V per (sequence, head) over a packed
// token sequence, the dominant cost of the MiniMax-H3 DiT block ("Buyer
// Questions: Current Evidence Status", Q4 current answer: attention is the
// largest share of the profiled block; "Open-H3-Regenerate-2K", forward table:
// dense attention on one B200).  Ragged batches follow "H3 Runtime Current
// State" (ragged sequence parallelism): each cu_seqlens segment attends only to
// itself, and CTAs take the segments longest first.  Dense launches may give
// the keys their own length (one block of a split key set: O and LSE are then
// that block's partial result; no keys at all give O = 0, LSE = -inf).
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
//   * warps 0-7 / 8-15 -- online softmax of Q0 / Q1.  A warp owns 16 tensor-
//     memory lanes and reads them with the 16x256b shape, so each query row's
//     128 scores sit in four threads of one warp (32 each): row maxima and sums
//     are two shuffles away, and two warps per scheduler work on each tile.  The
//     running max m (log2 units) may lag the true max by < 16, so P <= 2^16 and O
//     is rescaled in tensor memory only when the max grows by more.  The first
//     half of P is computed with m as it stands while the tile's maxima are
//     formed, and redone only when m must grow, so the max is off the step's
//     critical path;
//     p = 2^(s*c - m) with c = scale*log2(e), rounded to bf16 and stored over S
//     with the 16x128b shape; l sums the rounded weights the PV product uses
//     (they normalise to exactly one), lx the unrounded ones (log-sum-exp);
//   * epilogue by the softmax warps: O / l as bf16 (rows past the sequence end
//     are not stored); LSE = (m + log2 lx) * ln 2.
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
// log2 units: m is raised (and O rescaled) only when a row's maximum exceeds it by more
// than this, so P <= 2^16: far inside bf16 and fp32 range (O and l stay below
// n_keys * 2^16 * max|v|), and rows whose maximum creeps up in small steps (sharp
// softmax rows) rarely take the slow path.  A row whose running max is exact has its
// dominant weight exactly 1; with a lag that weight is rounded to bf16 like the rest.
constexpr float kRescaleThreshold = 16.0f;
constexpr int kSortMax = 256;              // ragged batches up to this many sequences run longest first

template <int D>
struct AttnTraits {
  static constexpr int kAtoms = D / 64;                      // 128-byte swizzle atoms along d
  static constexpr int kAtomBytes = kBM * 128;               // 128 rows x 128 bytes
  static constexpr int kTileBytes = kAtoms * kAtomBytes;     // one Q, K or V tile
  static constexpr int kStages = (D == 128) ? 4 : 8;         // K/V ring slots
  static constexpr int kTiles = kQTiles + kStages;
  // barriers: q, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], drain
  static constexpr int kBarriers = 1 + 2 * kStages + 3 * kQTiles + 1;
  static constexpr int kSmemBytes =
      1024 /*alignment slack*/ + kTiles * kTileBytes + 8 * kBarriers + 16 + 8 * kSortMax;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(256 + kQTiles * D <= 512, "tensor memory budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert((kTiles * kTileBytes) % 1024 == 0 && (8 * kBarriers) % 16 == 0, "barrier and scratch alignment");
};

struct AttnParams {
  uint16_t* o;                // bf16 output
  int64_t o_batch, o_tok, o_head;
  float* lse;                 // may be null
  const int32_t* cu_seqlens;  // ragged only
  int32_t nseq;               // ragged only
  int32_t n_heads;
  int64_t seqlen;             // dense: query tokens per sequence
  int64_t seqlen_kv;          // dense: key/value tokens per sequence (may differ, may be 0)
  int64_t total;              // ragged: total tokens (LSE row stride per head)
  // block-sparse (dense batches; null = every key tile): CSR lists of the key
  // tiles (kBN keys each) that each (batch, head, query-tile pair) sees, strictly
  // ascending; list (b * n_heads + h) * n_qpairs + pair
  const int32_t* blk_off;
  const int32_t* blk_idx;
  int64_t n_qpairs;
  float scale_log2;           // softmax_scale * log2(e)
  LaunchCtl ctl;
};

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
  const uint32_t bars = base + T::kTiles * T::kTileBytes;
  const uint32_t bar_q = bars;
  auto bar_kv_full = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_kv_empty = [&](int s) { return bars + 8u * (1 + kS + s); };
  auto bar_s_full = [&](int t) { return bars + 8u * (1 + 2 * kS + t); };
  auto bar_p_full = [&](int t) { return bars + 8u * (1 + 2 * kS + kQTiles + t); };
  auto bar_o_done = [&](int t) { return bars + 8u * (1 + 2 * kS + 2 * kQTiles + t); };
  const uint32_t bar_drain = bars + 8u * (1 + 2 * kS + 3 * kQTiles);  // MMA lane's exit after a failure
  volatile uint32_t* const slot_words =
      reinterpret_cast<volatile uint32_t*>(base_ptr + T::kTiles * T::kTileBytes + 8 * T::kBarriers);
  // slot_words[0] = tensor-memory base, [1] = work valid, [2] = sequence, [3] = query-pair index,
  // then the ragged scheduler's scratch (2 x kSortMax ints)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LaunchCtl ctl = p.ctl;

  // ---- ragged descriptor check (before anything reads a sequence bound) -------------
  // cu_seqlens[0] = 0, non-decreasing, no sequence longer than max_seqlen (p.seqlen,
  // which sized the grid) and cu_seqlens[nseq] = total.  Every CTA reaches the same
  // decision; a descriptor that breaks a rule is reported in the sticky error bits
  // and the launch writes nothing.
  if (kVarlen) {
    bool bad = false;
    for (int i = threadIdx.x; i < p.nseq; i += blockDim.x) {
      const int64_t a = __ldg(p.cu_seqlens + i), b = __ldg(p.cu_seqlens + i + 1);
      bad |= b < a || b - a > p.seqlen;
    }
    if (threadIdx.x == 0)
      bad |= __ldg(p.cu_seqlens) != 0 || static_cast<int64_t>(__ldg(p.cu_seqlens + p.nseq)) != p.total;
    if (__syncthreads_or(bad ? 1 : 0)) {
      if (threadIdx.x == 0) report_error(kErrBadSeqlens);
      return;  // CTA-uniform
    }
  }

  // ---- work decode (CTA-uniform, published through shared memory) ----------------
  // Ragged batches: the query-tile pairs of all sequences are numbered longest
  // sequence first (FLOPs grow with the square of the length, so the last CTAs of
  // the launch are the cheapest); with more than kSortMax sequences, in given order.
  int32_t* const sched = reinterpret_cast<int32_t*>(
      const_cast<uint32_t*>(slot_words) + 4);  // [kSortMax] lengths, then [kSortMax] order
  if (kVarlen && p.nseq <= kSortMax) {
    const int n = p.nseq;
    if (threadIdx.x < n) sched[threadIdx.x] = p.cu_seqlens[threadIdx.x + 1] - p.cu_seqlens[threadIdx.x];
    __syncthreads();
    if (threadIdx.x < n) {
      const int32_t mine = sched[threadIdx.x];
      int rank = 0;
      for (int i = 0; i < n; ++i) {
        const int32_t other = sched[i];
        rank += (other > mine || (other == mine && i < static_cast<int>(threadIdx.x))) ? 1 : 0;
      }
      sched[kSortMax + rank] = static_cast<int32_t>(threadIdx.x);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    uint32_t valid = launch_failed(ctl) ? 0u : 1u;
    uint32_t seq = 0, pair = blockIdx.x;
    if (kVarlen && valid) {
      valid = 0;
      uint32_t x = blockIdx.x;
      const bool sorted = p.nseq <= kSortMax;
      for (int i = 0; i < p.nseq; ++i) {
        const int s = sorted ? sched[kSortMax + i] : i;
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
  const int64_t kv_len = kVarlen ? seq_len : p.seqlen_kv;  // keys this sequence's queries see
  int nkv = static_cast<int>((kv_len + kBN - 1) / kBN);
  int kv_last_valid = static_cast<int>(kv_len - static_cast<int64_t>(nkv - 1) * kBN);
  // block-sparse: the tile loops below run over the listed key tiles; a list that
  // is not strictly ascending inside [0, nkv) is reported in the sticky error bits
  // and its CTA writes nothing (the other CTAs of the launch carry on)
  const int32_t* kv_list = nullptr;
  if (!kVarlen && p.blk_off != nullptr) {
    const int64_t c = (static_cast<int64_t>(batch) * p.n_heads + head) * p.n_qpairs + slot_words[3];
    const int32_t e0 = __ldg(p.blk_off + c), e1 = __ldg(p.blk_off + c + 1);
    const int cnt = e1 - e0;
    kv_list = p.blk_idx + e0;
    bool bad = cnt < 0 || cnt > nkv;
    for (int e = threadIdx.x; !bad && e < cnt; e += blockDim.x) {
      const int32_t x = __ldg(kv_list + e);
      bad = x < 0 || x >= nkv || (e > 0 && __ldg(kv_list + e - 1) >= x);
    }
    if (__syncthreads_or(bad ? 1 : 0)) {
      if (threadIdx.x == 0) report_error(kErrBadBlockList);
      return;  // CTA-uniform
    }
    if (cnt > 0 && __ldg(kv_list + cnt - 1) != nkv - 1) kv_last_valid = kBN;  // the ragged tile is not listed
    nkv = cnt;
  }
  if (nkv == 0) {
    // no keys (a block of a split key set may be empty): the empty sum, O = 0 and
    // LSE = -inf, for the CTA's rows; nothing else runs
    const int64_t row = q_row0 + threadIdx.x;
    if (threadIdx.x < kQTiles * kBM && row < seq_len &&
        store_in_bounds(seq_base + row < (kVarlen ? p.total : p.seqlen) && head < p.n_heads &&
                        batch < static_cast<int>(gridDim.z))) {
      uint4* orow = reinterpret_cast<uint4*>(p.o + static_cast<int64_t>(batch) * p.o_batch +
                                             (seq_base + row) * p.o_tok + static_cast<int64_t>(head) * p.o_head);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
      if (kLse) {
        float* lrow = kVarlen ? p.lse + static_cast<int64_t>(head) * p.total + seq_base
                              : p.lse + (static_cast<int64_t>(batch) * p.n_heads + head) * p.seqlen;
        lrow[row] = -INFINITY;
      }
    }
    return;
  }

  // ---- setup: barriers and tensor memory --------------------------------------------
  if (warp == kLoadWarp && lane == 0) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < kS; ++s) {
      ptx::mbar_init(bar_kv_full(s), 1);
      ptx::mbar_init(bar_kv_empty(s), 1);
    }
    for (int t = 0; t < kQTiles; ++t) {
      ptx::mbar_init(bar_s_full(t), 1);
      ptx::mbar_init(bar_p_full(t), kSoftmaxWarps / kQTiles);  // one arrival per warp of the tile
      ptx::mbar_init(bar_o_done(t), 1);
    }
    ptx::mbar_init(bar_drain, 1);
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
        const int32_t y_kv = y_seq + (kv_list ? __ldg(kv_list + j) : j) * kBN;
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
                             a * 64, y_kv, head, batch);
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
        mbar_wait_for(bar_q, 0, kDrainLimitNs);
        const uint32_t first = it > static_cast<uint32_t>(kS) ? it - kS : 0u;
        for (uint32_t u = first; u < it; ++u)
          mbar_wait_for(bar_kv_full(static_cast<int>(u % kS)), (u / kS) & 1u, kDrainLimitNs);
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

      // Descriptor sets for one K = 128 block, built while the thread waits anyway,
      // so each group of MMAs goes out back to back (d = 128: eight per group).
      auto q_descs = [&](int t, uint64_t (&d)[8]) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          d[kk] = ptx::sdesc_make(q_lo0 + t * kTile16 + (((kk >> 2) * T::kAtomBytes + (kk & 3) * 32) >> 4), kHi);
      };
      auto k_descs = [&](int ks, uint64_t (&d)[8]) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          d[kk] = ptx::sdesc_make(k_lo0 + ks * kTile16 + (((kk >> 2) * T::kAtomBytes + (kk & 3) * 32) >> 4), kHi);
      };
      auto v_descs = [&](int vs, uint64_t (&d)[8]) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) d[kk] = ptx::sdesc_make(v_lo0 + vs * kTile16 + ((kk * 16 * 128) >> 4), kHi);
      };
      auto p_addrs = [&](int t, uint32_t (&a)[8]) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) a[kk] = tmem + t * 128 + kk * 8;
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
        if constexpr (D == 128) {
          uint64_t dv[8], dk[8], dq[8];
          uint32_t ap[8];
          v_descs(slot_of(uv), dv);
          k_descs(slot_of(uk), dk);
#pragma unroll
          for (int t = 0; t < kQTiles; ++t) {
            q_descs(t, dq);
            p_addrs(t, ap);
            if (!mbar_wait(bar_p_full(t), static_cast<uint32_t>(j) & 1u, ctl)) { ok = false; break; }
            ptx::tc_fence_after();
            ptx::mma_ts_x8(tmem + 256 + t * D, ap, dv, kIdescPV, j > 0 ? 1u : 0u);
            ptx::mma_commit(bar_o_done(t));
            if (t == kQTiles - 1) ptx::mma_commit(bar_kv_empty(slot_of(uv)));
            if (has_next) {
              // K_{j+1} is only needed here, after PV_t(j) has been issued
              if (t == 0 && !mbar_wait(bar_kv_full(slot_of(uk)), parity_of(uk), ctl)) { ok = false; break; }
              ptx::mma_ss_x8(tmem + t * 128, dq, dk, kIdescQK, 0u);
              ptx::mma_commit(bar_s_full(t));
            }
          }
        } else {
          for (int t = 0; t < kQTiles; ++t) {
            if (!mbar_wait(bar_p_full(t), static_cast<uint32_t>(j) & 1u, ctl)) { ok = false; break; }
            ptx::tc_fence_after();
            issue_pv(t, slot_of(uv), j == 0);
            if (t == kQTiles - 1) ptx::mma_commit(bar_kv_empty(slot_of(uv)));
            if (has_next) {
              if (t == 0 && !mbar_wait(bar_kv_full(slot_of(uk)), parity_of(uk), ctl)) { ok = false; break; }
              issue_s(t, slot_of(uk));
            }
          }
        }
        if (!ok) break;
        if (has_next) ptx::mma_commit(bar_kv_empty(slot_of(uk)));
      }
      if (!ok) {
        // failure: every MMA already issued must finish writing tensor memory
        // before the teardown frees it (the next CTA on this SM may own it then)
        ptx::mma_commit(bar_drain);
        mbar_wait_for(bar_drain, 0, kDrainLimitNs);
      }
    }
  } else {
    // ============================ softmax + epilogue ==============================
    // Warps 0-7 serve tile 0 and warps 8-15 tile 1.  A warp owns 16 tensor-memory
    // lanes (half of its lane quarter) and reads them with the 16x256b shape:
    // thread t holds rows r0 = t/4 and r1 = t/4 + 8 of those 16, 32 keys each
    // (columns 8k + 2(t%4) + {0,1}), so a row's 128 keys sit in 4 threads of the
    // same warp and its max and sums are two shuffles away.
    const int t = warp >> 3;                 // query tile
    const int quarter = warp & 3;
    const int lhalf = (warp >> 2) & 1;       // which 16 lanes of the quarter
    const int cq = lane & 3;                 // column phase inside each 8-column chunk
    const int lane0 = quarter * 32 + lhalf * 16;   // first tensor-memory lane of this warp
    const int r0 = lane0 + (lane >> 2);      // this thread's two rows (tile-relative)
    const int r1 = r0 + 8;
    const uint32_t lane_off = static_cast<uint32_t>(lane0) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const float c = p.scale_log2;
    const float2 c2 = make_float2(c, c);
    float m0 = -INFINITY, m1 = -INFINITY;  // running row maxima of s*c (log2), may lag by < 16
    float l0 = 0.0f, l1 = 0.0f;            // this thread's partial sums of bf16(2^(s*c - m))
    float lx0 = 0.0f, lx1 = 0.0f;          // the same in fp32 (log-sum-exp)
    bool ok = true;

    for (int j = 0; j < nkv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(t), static_cast<uint32_t>(j) & 1u, ctl));
      if (!ok) break;
      ptx::tc_fence_after();
      // s0[e] / s1[e], e = 2k + i, is the score of key 8k + 2*cq + i for row r0 / r1
      float s0[32], s1[32];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        uint32_t r[32];
        ptx::tmem_ld_16x256b_x8(tS + hb * 64, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int k = hb * 8 + kk;
          s0[2 * k] = __uint_as_float(r[4 * kk]);
          s0[2 * k + 1] = __uint_as_float(r[4 * kk + 1]);
          s1[2 * k] = __uint_as_float(r[4 * kk + 2]);
          s1[2 * k + 1] = __uint_as_float(r[4 * kk + 3]);
        }
      }
      if (j == nkv - 1 && kv_last_valid < kBN) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = 8 * (e >> 1) + 2 * cq + (e & 1);
          if (key >= kv_last_valid) s0[e] = s1[e] = -INFINITY;
        }
      }
      // P = 2^(s*c - m) rounded to bf16, stored over S as packed pairs: the pair of
      // keys 8k + 2*cq + {0,1} is packed column 4k + cq (16x128b shape).
      float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
      float2 accx0 = make_float2(0.0f, 0.0f), accx1 = make_float2(0.0f, 0.0f);
      // one pair of keys for both rows: exponentials, packing, sums
      auto p_pair = [&](float sa0, float sa1, float sb0, float sb1, float2 nm0, float2 nm1, uint32_t& pa,
                        uint32_t& pb) {
        const float2 x0 = __ffma2_rn(make_float2(sa0, sa1), c2, nm0);
        const float2 x1 = __ffma2_rn(make_float2(sb0, sb1), c2, nm1);
        const float2 e0 = make_float2(ptx::ex2_approx(x0.x), ptx::ex2_approx(x0.y));
        const float2 e1 = make_float2(ptx::ex2_approx(x1.x), ptx::ex2_approx(x1.y));
        pa = ptx::pack_bf16x2(e0.x, e0.y);
        pb = ptx::pack_bf16x2(e1.x, e1.y);
        ptx::add_bf16x2_f32(acc0.x, acc0.y, pa);
        ptx::add_bf16x2_f32(acc1.x, acc1.y, pb);
        if (kLse) {
          accx0 = __fadd2_rn(accx0, e0);
          accx1 = __fadd2_rn(accx1, e1);
        }
      };
      uint32_t pk[16];
      // First half (keys 0..63) with the running max m as it stands, while this
      // tile's row maxima are formed beside it on another pipe (the max chains are
      // interleaved with the exponentials in the issue order).  Only where a max
      // grows by more than the threshold (always at j = 0, rarely later) are m and
      // that half redone, so the max is off the critical path of the step.
      float a0 = fmaxf(s0[0], s0[1]), b0 = fmaxf(s0[2], s0[3]);
      float a1 = fmaxf(s1[0], s1[1]), b1 = fmaxf(s1[2], s1[3]);
      {
        const float2 nm0 = make_float2(-m0, -m0), nm1 = make_float2(-m1, -m1);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          p_pair(s0[2 * k], s0[2 * k + 1], s1[2 * k], s1[2 * k + 1], nm0, nm1, pk[2 * k], pk[2 * k + 1]);
          if (k < 7) {
            const int e = 4 * (k + 1);
            a0 = ptx::max3(a0, s0[e], s0[e + 1]);
            b0 = ptx::max3(b0, s0[e + 2], s0[e + 3]);
            a1 = ptx::max3(a1, s1[e], s1[e + 1]);
            b1 = ptx::max3(b1, s1[e + 2], s1[e + 3]);
          }
        }
      }
      // row maxima: this thread's 32 keys (above), then the quad's four threads
      float mx0 = fmaxf(a0, b0), mx1 = fmaxf(a1, b1);
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float cand0 = mx0 * c, cand1 = mx1 * c;
      const bool grow0 = cand0 > m0 + kRescaleThreshold;  // identical in the row's 4 threads
      const bool grow1 = cand1 > m1 + kRescaleThreshold;
      float alpha0 = 1.0f, alpha1 = 1.0f;
      const bool any_grow = __any_sync(0xffffffffu, grow0 || grow1);
      if (any_grow) {
        if (grow0) {
          alpha0 = ptx::ex2_approx(m0 - cand0);
          m0 = cand0;
        }
        if (grow1) {
          alpha1 = ptx::ex2_approx(m1 - cand1);
          m1 = cand1;
        }
        // redo the first half from the scores still in tensor memory (P has not
        // been stored over them yet), 32 columns at a time to spare registers
        acc0 = acc1 = accx0 = accx1 = make_float2(0.0f, 0.0f);
        const float2 nm0 = make_float2(-m0, -m0), nm1 = make_float2(-m1, -m1);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t r[16];
          ptx::tmem_ld_16x256b_x4(tS + ch * 32, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = ch * 4 + kk;
            float v[4] = {__uint_as_float(r[4 * kk]), __uint_as_float(r[4 * kk + 1]),
                          __uint_as_float(r[4 * kk + 2]), __uint_as_float(r[4 * kk + 3])};
            if (j == nkv - 1) {
#pragma unroll
              for (int i = 0; i < 2; ++i)
                if (8 * k + 2 * cq + i >= kv_last_valid) v[i] = v[2 + i] = -INFINITY;
            }
            p_pair(v[0], v[1], v[2], v[3], nm0, nm1, pk[2 * k], pk[2 * k + 1]);
          }
        }
      }
      ptx::tmem_st_16x128b_x8(tS, pk);
      // second half (keys 64..127) with the final m
      {
        const float2 nm0 = make_float2(-m0, -m0), nm1 = make_float2(-m1, -m1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int k = 8 + kk;
          p_pair(s0[2 * k], s0[2 * k + 1], s1[2 * k], s1[2 * k + 1], nm0, nm1, pk[2 * kk], pk[2 * kk + 1]);
        }
      }
      ptx::tmem_st_16x128b_x8(tS + 32, pk);
      l0 = l0 * alpha0 + (acc0.x + acc0.y);
      l1 = l1 * alpha1 + (acc1.x + acc1.y);
      if (kLse) {
        lx0 = lx0 * alpha0 + (accx0.x + accx0.y);
        lx1 = lx1 * alpha1 + (accx1.x + accx1.y);
      }
      if (j > 0 && any_grow) {
        // O_t(j-1) is final once S_t(j) has landed (the tensor core runs in issue
        // order); the explicit wait keeps that visible.  Rescale it in place.
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done(t), static_cast<uint32_t>(j - 1) & 1u, ctl));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int hb = 0; hb < D / 64; ++hb) {
          uint32_t r[32];
          ptx::tmem_ld_16x256b_x8(tO + hb * 64, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            r[4 * kk] = __float_as_uint(__uint_as_float(r[4 * kk]) * alpha0);
            r[4 * kk + 1] = __float_as_uint(__uint_as_float(r[4 * kk + 1]) * alpha0);
            r[4 * kk + 2] = __float_as_uint(__uint_as_float(r[4 * kk + 2]) * alpha1);
            r[4 * kk + 3] = __float_as_uint(__uint_as_float(r[4 * kk + 3]) * alpha1);
          }
          ptx::tmem_st_16x256b_x8(tO + hb * 64, r);
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
      // a row's sums: add the quad's partials
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      ptx::tc_fence_after();
      const int64_t row0 = q_row0 + t * kBM + r0, row1 = q_row0 + t * kBM + r1;  // within the sequence
      const int64_t tok_extent = kVarlen ? p.total : p.seqlen;  // token rows of O and of each LSE row
      const bool in_launch = head < p.n_heads && batch < static_cast<int>(gridDim.z);
      const bool v0 = row0 < seq_len && store_in_bounds(in_launch && seq_base + row0 < tok_extent);
      const bool v1 = row1 < seq_len && store_in_bounds(in_launch && seq_base + row1 < tok_extent);
      const float inv0 = 1.0f / l0, inv1 = 1.0f / l1;
      uint16_t* const obase = p.o + static_cast<int64_t>(batch) * p.o_batch + static_cast<int64_t>(head) * p.o_head;
      uint32_t* const o0 = reinterpret_cast<uint32_t*>(obase + (seq_base + row0) * p.o_tok) + cq;
      uint32_t* const o1 = reinterpret_cast<uint32_t*>(obase + (seq_base + row1) * p.o_tok) + cq;
#pragma unroll
      for (int hb = 0; hb < D / 64; ++hb) {
        uint32_t r[32];
        ptx::tmem_ld_16x256b_x8(tO + hb * 64, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int k = hb * 8 + kk;  // columns 8k + 2*cq + {0,1}: the 32-bit word 4k + cq
          if (v0) o0[4 * k] = ptx::pack_bf16x2(__uint_as_float(r[4 * kk]) * inv0, __uint_as_float(r[4 * kk + 1]) * inv0);
          if (v1) o1[4 * k] = ptx::pack_bf16x2(__uint_as_float(r[4 * kk + 2]) * inv1, __uint_as_float(r[4 * kk + 3]) * inv1);
        }
      }
      if (kLse) {
        lx0 += __shfl_xor_sync(0xffffffffu, lx0, 1);
        lx1 += __shfl_xor_sync(0xffffffffu, lx1, 1);
        lx0 += __shfl_xor_sync(0xffffffffu, lx0, 2);
        lx1 += __shfl_xor_sync(0xffffffffu, lx1, 2);
        if (cq == 0) {
          const float ln2 = 0.69314718055994530942f;
          if (kVarlen) {
            float* lrow = p.lse + static_cast<int64_t>(head) * p.total + seq_base;
            if (v0) lrow[row0] = (m0 + log2f(lx0)) * ln2;
            if (v1) lrow[row1] = (m1 + log2f(lx1)) * ln2;
          } else {
            float* lrow = p.lse + (static_cast<int64_t>(batch) * p.n_heads + head) * p.seqlen;
            if (v0) lrow[row0] = (m0 + log2f(lx0)) * ln2;
            if (v1) lrow[row1] = (m1 + log2f(lx1)) * ln2;
          }
        }
      }
    }
  }

  // ---- teardown: every thread arrives here, then the allocating warp frees TMEM ----
  if (warp < kSoftmaxWarps) ptx::tmem_wait_st();  // a softmax warp that left early may have stores in flight
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, T::kTmemCols);
  }
}

}  // namespace h3
