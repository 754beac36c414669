// h3attn_api.cu -- the C ABI declared in include/h3attn.h: argument checks,
// TMA tensor-map encoding, launch configuration, and the device error word.
//
// The whole library is this one translation unit (the kernels come in through
// the headers), so it needs no relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "h3attn.h"

#include "attention.cuh"
#include "common.cuh"
#include "merge.cuh"
#include "prologue.cuh"
#include "qkv.cuh"
#include "selftest.cuh"

namespace {

// The projection runs as CTA pairs (M256 tiles across two SMs) unless built
// with H3_QKV_PAIRS=0.
#ifndef H3_QKV_PAIRS
#define H3_QKV_PAIRS 1
#endif
constexpr bool kQkvPairs = H3_QKV_PAIRS != 0;

constexpr int kVersion = 10000;  // 1.0.0

thread_local char t_last_error[512] = "";

h3attn_status fail(h3attn_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

h3attn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(H3ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s) { return s > 0 && (s % 8) == 0; }

std::atomic<uint32_t> g_launch_counter{0};
uint32_t next_launch_id() {
  uint32_t id;
  do {
    id = g_launch_counter.fetch_add(1, std::memory_order_relaxed) + 1u;
  } while (id == 0u);
  return id;
}

// ---- driver entry point for cuTensorMapEncodeTiled (no link against libcuda) ----------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    }
  });
  return fn;
}

// A bf16 [B][N][H][D] view (token-major) as a 4D tensor map with 128-row x 64-element
// boxes and 128-byte swizzle.  Token rows outside [0, N) read as zeros.
h3attn_status make_map(CUtensorMap* map, const void* ptr, int d, int64_t n_tok, int n_heads,
                       int64_t n_batch, int64_t s_tok, int64_t s_head, int64_t s_batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(H3ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n_tok),
                        static_cast<cuuint64_t>(n_heads), static_cast<cuuint64_t>(n_batch)};
  if (n_batch == 1) s_batch = s_tok;  // extent 1: the stride is never used
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s_tok) * 2, static_cast<cuuint64_t>(s_head) * 2,
                           static_cast<cuuint64_t>(s_batch) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(h3::kBM), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(H3ATTN_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return H3ATTN_OK;
}

// Per-device one-time kernel attributes (dynamic shared memory opt-in).
template <typename K>
cudaError_t ensure_smem_attr(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, bool kVarlen>
h3attn_status launch_attention(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                               const h3::AttnParams& prm, dim3 grid, cudaStream_t stream) {
  using T = h3::AttnTraits<D>;
  auto kernel = prm.lse ? h3::attn_fwd_kernel<D, kVarlen, true> : h3::attn_fwd_kernel<D, kVarlen, false>;
  cudaError_t e = ensure_smem_attr(kernel, T::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attention)");
  kernel<<<grid, h3::kAttnThreads, T::kSmemBytes, stream>>>(mq, mk, mv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return H3ATTN_OK;
}

h3attn_status check_common(const void* q, const void* k, const void* v, void* o, int32_t n_heads,
                           int32_t head_dim) {
  if (!q || !k || !v || !o) return fail(H3ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (n_heads <= 0 || n_heads > 65535) return fail(H3ATTN_ERR_INVALID_ARG, "n_heads must be in [1, 65535]");
  if (head_dim != 64 && head_dim != 128)
    return fail(H3ATTN_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(H3ATTN_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  return H3ATTN_OK;
}

h3attn_status check_strides(const int64_t* s, int n, const char* name) {
  if (!s) return fail(H3ATTN_ERR_INVALID_ARG, "%s strides are null", name);
  for (int i = 0; i < n; ++i) {
    if (s[i] <= 0) return fail(H3ATTN_ERR_INVALID_ARG, "%s stride %d must be positive", name, i);
    if (s[i] % 8 != 0) return fail(H3ATTN_ERR_MISALIGNED, "%s stride %d not a multiple of 8 elements", name, i);
    if (s[i] >= (int64_t(1) << 38)) return fail(H3ATTN_ERR_UNSUPPORTED, "%s stride %d too large", name, i);
  }
  return H3ATTN_OK;
}

// Rotary tables shared by the prologue and the fused projection: pair p of the 3D
// layout belongs to section ax at pair index i inside it, with frequency
// theta^(-2i/width); 1D tokens use theta^(-2p/d) over all pairs.
h3attn_status rope_tables(h3::RopeTables* rope, const uint8_t* kind, int head_dim, int sec_t, int sec_h,
                          int sec_w, double theta) {
  if (!kind) return fail(H3ATTN_ERR_INVALID_ARG, "kind is required with pos");
  if (sec_t < 0 || sec_h < 0 || sec_w < 0 || (sec_t | sec_h | sec_w) & 1 || sec_t + sec_h + sec_w != head_dim)
    return fail(H3ATTN_ERR_INVALID_ARG, "sections %d/%d/%d must be even and sum to head_dim %d", sec_t, sec_h,
                sec_w, head_dim);
  if (!(theta > 0.0) || !std::isfinite(theta)) return fail(H3ATTN_ERR_INVALID_ARG, "theta must be > 0");
  const int widths[3] = {sec_t, sec_h, sec_w};
  int pair = 0;
  for (int ax = 0; ax < 3; ++ax) {
    for (int i = 0; i < widths[ax] / 2; ++i, ++pair) {
      rope->axis_3d[pair] = static_cast<uint8_t>(ax);
      rope->inv_freq_3d[pair] = std::exp(-(2.0 * i / widths[ax]) * std::log(theta));
    }
  }
  for (int i = 0; i < head_dim / 2; ++i) rope->inv_freq_1d[i] = std::exp(-(2.0 * i / head_dim) * std::log(theta));
  return H3ATTN_OK;
}

// A row-major bf16 matrix [rows][cols] (row stride in elements) as a tensor map
// with 64-column x box_rows boxes and 128-byte swizzle (the K-major operand tiles
// of the projection GEMM).  Rows past the end read as zeros.
h3attn_status make_map_rows(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t row_stride,
                            int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(H3ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1, 1};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(row_stride) * 2, static_cast<cuuint64_t>(row_stride) * 2 * rows,
                           static_cast<cuuint64_t>(row_stride) * 2 * rows};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(H3ATTN_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return H3ATTN_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// How many CTA pairs (clusters of two) of a kernel fit on the device at once: the
// persistent grid of the paired projection.  Falls back to half the SMs.
int resident_pairs(const void* kernel, int smem_bytes) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2u * static_cast<unsigned>(sm_count()), 1, 1);
  cfg.blockDim = dim3(h3::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  return n;
}

float resolve_scale(float scale, int d) {
  const float s = scale > 0.0f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  return static_cast<float>(static_cast<double>(s) * 1.4426950408889634074);
}

// Dense batches of equal-length sequences (optionally a separate key length and
// block-sparse key lists): argument checks, tensor maps, launch.
h3attn_status fwd_dense(const void* q, const void* k, const void* v, void* o, int32_t batch, int64_t seqlen_q,
                        int64_t seqlen_kv, int32_t n_heads, int32_t head_dim, const int64_t q_strides[3],
                        const int64_t k_strides[3], const int64_t v_strides[3], const int64_t o_strides[3],
                        float softmax_scale, float* lse, const int32_t* blk_off, const int32_t* blk_idx,
                        void* stream) {
  if (seqlen_kv < 0) return fail(H3ATTN_ERR_INVALID_ARG, "seqlen_kv must not be negative");
  // with no keys, k and v are never read and may be null (an empty tensor's data pointer)
  const void* k_chk = (seqlen_kv == 0 && !k) ? q : k;
  const void* v_chk = (seqlen_kv == 0 && !v) ? q : v;
  h3attn_status st = check_common(q, k_chk, v_chk, o, n_heads, head_dim);
  if (st != H3ATTN_OK) return st;
  if (batch <= 0 || batch > 65535) return fail(H3ATTN_ERR_INVALID_ARG, "batch must be in [1, 65535]");
  if (seqlen_q <= 0) return fail(H3ATTN_ERR_INVALID_ARG, "seqlen must be positive");
  if (seqlen_q > (int64_t(1) << 30) || seqlen_kv > (int64_t(1) << 30))
    return fail(H3ATTN_ERR_UNSUPPORTED, "seqlen too large");
  if ((st = check_strides(q_strides, 3, "q")) != H3ATTN_OK) return st;
  if ((st = check_strides(k_strides, 3, "k")) != H3ATTN_OK) return st;
  if ((st = check_strides(v_strides, 3, "v")) != H3ATTN_OK) return st;
  if ((st = check_strides(o_strides, 3, "o")) != H3ATTN_OK) return st;
  if (!std::isfinite(softmax_scale)) return fail(H3ATTN_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(H3ATTN_ERR_MISALIGNED, "lse must be 4-byte aligned");

  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, head_dim, seqlen_q, n_heads, batch, q_strides[1], q_strides[2], q_strides[0])) != H3ATTN_OK) return st;
  if (seqlen_kv > 0) {
    if ((st = make_map(&mk, k, head_dim, seqlen_kv, n_heads, batch, k_strides[1], k_strides[2], k_strides[0])) != H3ATTN_OK) return st;
    if ((st = make_map(&mv, v, head_dim, seqlen_kv, n_heads, batch, v_strides[1], v_strides[2], v_strides[0])) != H3ATTN_OK) return st;
  } else {
    mk = mq;  // no keys: the kernel writes the empty result and reads neither map
    mv = mq;
  }

  h3::AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.o = static_cast<uint16_t*>(o);
  prm.o_batch = o_strides[0];
  prm.o_tok = o_strides[1];
  prm.o_head = o_strides[2];
  prm.lse = lse;
  prm.n_heads = n_heads;
  prm.seqlen = seqlen_q;
  prm.seqlen_kv = seqlen_kv;
  prm.total = seqlen_q;
  prm.scale_log2 = resolve_scale(softmax_scale, head_dim);
  prm.ctl.launch_id = next_launch_id();

  const int64_t pairs = (seqlen_q + h3::kQTiles * h3::kBM - 1) / (h3::kQTiles * h3::kBM);
  prm.blk_off = blk_off;
  prm.blk_idx = blk_idx;
  prm.n_qpairs = pairs;
  dim3 grid(static_cast<unsigned>(pairs), static_cast<unsigned>(n_heads), static_cast<unsigned>(batch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return head_dim == 128 ? launch_attention<128, false>(mq, mk, mv, prm, grid, s)
                         : launch_attention<64, false>(mq, mk, mv, prm, grid, s);
}

}  // namespace

extern "C" {

int h3attn_version(void) { return kVersion; }

int h3attn_build_flags(void) { return h3::kDebugBounds ? H3ATTN_BUILD_DEBUG_BOUNDS : 0; }

const char* h3attn_status_string(int status) {
  switch (status) {
    case H3ATTN_OK: return "ok";
    case H3ATTN_ERR_INVALID_ARG: return "invalid argument";
    case H3ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case H3ATTN_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case H3ATTN_ERR_CUDA: return "CUDA error";
    case H3ATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    default: return "unknown status";
  }
}

const char* h3attn_last_error(void) { return t_last_error; }

int h3attn_device_status(void* stream, int clear) {
  // The word is read and (with clear) zeroed by one atomic exchange on the device,
  // ordered after the stream's earlier work, so an error another stream records
  // meanwhile stays in the word for the next call.  The snapshot it is copied
  // through is shared, so concurrent calls in this process take turns.
  static std::mutex status_mutex;
  std::lock_guard<std::mutex> lock(status_mutex);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h3::status_exchange_kernel<<<1, 32, 0, st>>>(clear ? 1 : 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "status exchange launch");
  uint32_t word[2] = {0, 0};
  e = cudaMemcpyFromSymbolAsync(word, h3::g_status_snapshot, sizeof(word), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (word[0] & h3::kErrBounds)
    return fail(H3ATTN_ERR_INVALID_ARG,
                "a debug bounds check fired: a kernel computed a store index outside its launch's extents "
                "(the store was skipped)");
  if (word[0] & h3::kErrBadSeqlens)
    return fail(H3ATTN_ERR_INVALID_ARG,
                "cu_seqlens broke its rules (cu[0] = 0, non-decreasing, lengths <= max_seqlen, "
                "cu[nseq] = total_tokens); that launch wrote nothing");
  if (word[0] & h3::kErrBadBlockList)
    return fail(H3ATTN_ERR_INVALID_ARG, "a block-sparse key list was not strictly ascending in range");
  if (word[0] & h3::kErrTimeout)
    return fail(H3ATTN_ERR_DEVICE_TIMEOUT, "a kernel timed out on an internal barrier (launch %u)", word[1]);
  return H3ATTN_OK;
}

h3attn_status h3attn_selftest_wait_timeout(void* stream) {
  h3::LaunchCtl ctl;
  ctl.launch_id = next_launch_id();
  h3::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctl);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return H3ATTN_OK;
}

h3attn_status h3attn_prologue(const void* q_in, const void* k_in, void* q_out, void* k_out,
                              int64_t n_tokens, int32_t n_heads, int32_t head_dim,
                              int64_t in_tok_stride, int64_t in_head_stride,
                              int64_t out_tok_stride, int64_t out_head_stride,
                              const void* gamma_q, const void* gamma_k, double eps,
                              const int32_t* pos, const uint8_t* kind,
                              int32_t sec_t, int32_t sec_h, int32_t sec_w, double theta,
                              void* stream) {
  if (!q_in || !k_in || !q_out || !k_out) return fail(H3ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (n_tokens < 0) return fail(H3ATTN_ERR_INVALID_ARG, "n_tokens must be >= 0");
  if (n_heads <= 0) return fail(H3ATTN_ERR_INVALID_ARG, "n_heads must be positive");
  if (head_dim != 64 && head_dim != 128)
    return fail(H3ATTN_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) ||
      (gamma_q && !aligned16(gamma_q)) || (gamma_k && !aligned16(gamma_k)))
    return fail(H3ATTN_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  const int64_t strides[4] = {in_tok_stride, in_head_stride, out_tok_stride, out_head_stride};
  h3attn_status st = check_strides(strides, 4, "prologue");
  if (st != H3ATTN_OK) return st;
  if (!(eps >= 0.0) || !std::isfinite(eps)) return fail(H3ATTN_ERR_INVALID_ARG, "eps must be finite and >= 0");

  h3::PrologueParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (pos && (st = rope_tables(&prm.rope, kind, head_dim, sec_t, sec_h, sec_w, theta)) != H3ATTN_OK) return st;
  if (n_tokens == 0) return H3ATTN_OK;
  prm.q_in = static_cast<const uint16_t*>(q_in);
  prm.k_in = static_cast<const uint16_t*>(k_in);
  prm.q_out = static_cast<uint16_t*>(q_out);
  prm.k_out = static_cast<uint16_t*>(k_out);
  prm.n_tokens = n_tokens;
  prm.in_tok = in_tok_stride;
  prm.in_head = in_head_stride;
  prm.out_tok = out_tok_stride;
  prm.out_head = out_head_stride;
  prm.gamma_q = static_cast<const uint16_t*>(gamma_q);
  prm.gamma_k = static_cast<const uint16_t*>(gamma_k);
  prm.pos = pos;
  prm.kind = kind;
  prm.n_heads = n_heads;
  prm.eps = static_cast<float>(eps);

  constexpr int kThreads = h3::kPrologueThreads;
  constexpr int kTokensPerBlock = kThreads / 32;  // one warp per token
  const int64_t blocks = (n_tokens + kTokensPerBlock - 1) / kTokensPerBlock;
  if (blocks > 0x7FFFFFFF) return fail(H3ATTN_ERR_UNSUPPORTED, "too many tokens");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 128) {
    h3::prologue_kernel<128><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(prm);
  } else {
    h3::prologue_kernel<64><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(prm);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
  return H3ATTN_OK;
}

h3attn_status h3attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, int32_t batch,
                                      int64_t seqlen_q, int64_t seqlen_kv, int32_t n_heads, int32_t head_dim,
                                      const int64_t q_strides[3], const int64_t k_strides[3],
                                      const int64_t v_strides[3], const int64_t o_strides[3],
                                      const int32_t* blk_off, const int32_t* blk_idx, float softmax_scale,
                                      float* lse, void* stream) {
  if (!blk_off || !blk_idx) return fail(H3ATTN_ERR_INVALID_ARG, "null block list");
  if ((reinterpret_cast<uintptr_t>(blk_off) | reinterpret_cast<uintptr_t>(blk_idx)) & 3u)
    return fail(H3ATTN_ERR_MISALIGNED, "block lists must be 4-byte aligned");
  return fwd_dense(q, k, v, o, batch, seqlen_q, seqlen_kv, n_heads, head_dim, q_strides, k_strides, v_strides,
                   o_strides, softmax_scale, lse, blk_off, blk_idx, stream);
}

h3attn_status h3attn_fwd_kv(const void* q, const void* k, const void* v, void* o, int32_t batch,
                            int64_t seqlen_q, int64_t seqlen_kv, int32_t n_heads, int32_t head_dim,
                            const int64_t q_strides[3], const int64_t k_strides[3],
                            const int64_t v_strides[3], const int64_t o_strides[3], float softmax_scale,
                            float* lse, void* stream) {
  return fwd_dense(q, k, v, o, batch, seqlen_q, seqlen_kv, n_heads, head_dim, q_strides, k_strides, v_strides,
                   o_strides, softmax_scale, lse, nullptr, nullptr, stream);
}

h3attn_status h3attn_fwd(const void* q, const void* k, const void* v, void* o, int32_t batch,
                         int64_t seqlen, int32_t n_heads, int32_t head_dim, const int64_t q_strides[3],
                         const int64_t k_strides[3], const int64_t v_strides[3],
                         const int64_t o_strides[3], float softmax_scale, float* lse, void* stream) {
  if (seqlen <= 0) return fail(H3ATTN_ERR_INVALID_ARG, "seqlen must be positive");
  return h3attn_fwd_kv(q, k, v, o, batch, seqlen, seqlen, n_heads, head_dim, q_strides, k_strides, v_strides,
                       o_strides, softmax_scale, lse, stream);
}

h3attn_status h3attn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b, void* o,
                           float* lse, int32_t batch, int64_t seqlen, int32_t n_heads, int32_t head_dim,
                           const int64_t oa_strides[3], const int64_t ob_strides[3],
                           const int64_t o_strides[3], void* stream) {
  if (!o_a || !o_b || !o || !lse_a || !lse_b || !lse) return fail(H3ATTN_ERR_INVALID_ARG, "null pointer");
  if (head_dim != 64 && head_dim != 128)
    return fail(H3ATTN_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (batch <= 0 || batch > 65535) return fail(H3ATTN_ERR_INVALID_ARG, "batch must be in [1, 65535]");
  if (n_heads <= 0 || n_heads > 65535) return fail(H3ATTN_ERR_INVALID_ARG, "n_heads must be in [1, 65535]");
  if (seqlen < 0 || seqlen > (int64_t(1) << 30)) return fail(H3ATTN_ERR_INVALID_ARG, "seqlen must be in [0, 2^30]");
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o))
    return fail(H3ATTN_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(lse_a) | reinterpret_cast<uintptr_t>(lse_b) | reinterpret_cast<uintptr_t>(lse)) & 3u)
    return fail(H3ATTN_ERR_MISALIGNED, "lse arrays must be 4-byte aligned");
  h3attn_status st;
  if ((st = check_strides(oa_strides, 3, "o_a")) != H3ATTN_OK) return st;
  if ((st = check_strides(ob_strides, 3, "o_b")) != H3ATTN_OK) return st;
  if ((st = check_strides(o_strides, 3, "o")) != H3ATTN_OK) return st;
  if (seqlen == 0) return H3ATTN_OK;

  h3::MergeParams prm;
  prm.oa = static_cast<const uint16_t*>(o_a);
  prm.ob = static_cast<const uint16_t*>(o_b);
  prm.o = static_cast<uint16_t*>(o);
  prm.oa_batch = oa_strides[0]; prm.oa_tok = oa_strides[1]; prm.oa_head = oa_strides[2];
  prm.ob_batch = ob_strides[0]; prm.ob_tok = ob_strides[1]; prm.ob_head = ob_strides[2];
  prm.o_batch = o_strides[0]; prm.o_tok = o_strides[1]; prm.o_head = o_strides[2];
  prm.lse_a = lse_a;
  prm.lse_b = lse_b;
  prm.lse = lse;
  prm.seqlen = seqlen;
  prm.n_heads = n_heads;
  dim3 grid(static_cast<unsigned>((seqlen + h3::kMergeTokens - 1) / h3::kMergeTokens),
            static_cast<unsigned>(n_heads), static_cast<unsigned>(batch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 128) {
    h3::merge_kernel<128><<<grid, h3::kMergeThreads, 0, s>>>(prm);
  } else {
    h3::merge_kernel<64><<<grid, h3::kMergeThreads, 0, s>>>(prm);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return H3ATTN_OK;
}

h3attn_status h3attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                const int32_t* cu_seqlens, int32_t nseq, int64_t total_tokens,
                                int32_t max_seqlen, int32_t n_heads, int32_t head_dim,
                                const int64_t q_strides[2], const int64_t k_strides[2],
                                const int64_t v_strides[2], const int64_t o_strides[2],
                                float softmax_scale, float* lse, void* stream) {
  h3attn_status st = check_common(q, k, v, o, n_heads, head_dim);
  if (st != H3ATTN_OK) return st;
  if (!cu_seqlens) return fail(H3ATTN_ERR_INVALID_ARG, "cu_seqlens is null");
  if (nseq <= 0 || nseq > 65535) return fail(H3ATTN_ERR_INVALID_ARG, "nseq must be in [1, 65535]");
  if (total_tokens <= 0 || total_tokens > (int64_t(1) << 30))
    return fail(H3ATTN_ERR_INVALID_ARG, "total_tokens must be in [1, 2^30]");
  if (max_seqlen <= 0 || max_seqlen > total_tokens)
    return fail(H3ATTN_ERR_INVALID_ARG, "max_seqlen must be in [1, total_tokens]");
  if ((st = check_strides(q_strides, 2, "q")) != H3ATTN_OK) return st;
  if ((st = check_strides(k_strides, 2, "k")) != H3ATTN_OK) return st;
  if ((st = check_strides(v_strides, 2, "v")) != H3ATTN_OK) return st;
  if ((st = check_strides(o_strides, 2, "o")) != H3ATTN_OK) return st;
  if (!std::isfinite(softmax_scale)) return fail(H3ATTN_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(H3ATTN_ERR_MISALIGNED, "lse must be 4-byte aligned");

  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, head_dim, total_tokens, n_heads, 1, q_strides[0], q_strides[1], 0)) != H3ATTN_OK) return st;
  if ((st = make_map(&mk, k, head_dim, total_tokens, n_heads, 1, k_strides[0], k_strides[1], 0)) != H3ATTN_OK) return st;
  if ((st = make_map(&mv, v, head_dim, total_tokens, n_heads, 1, v_strides[0], v_strides[1], 0)) != H3ATTN_OK) return st;

  h3::AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.o = static_cast<uint16_t*>(o);
  prm.o_batch = 0;
  prm.o_tok = o_strides[0];
  prm.o_head = o_strides[1];
  prm.lse = lse;
  prm.cu_seqlens = cu_seqlens;
  prm.nseq = nseq;
  prm.n_heads = n_heads;
  prm.seqlen = max_seqlen;
  prm.total = total_tokens;
  prm.scale_log2 = resolve_scale(softmax_scale, head_dim);
  prm.ctl.launch_id = next_launch_id();

  // upper bound on query-tile pairs: each sequence wastes at most one partial pair, and
  // none has more than ceil(max_seqlen / 256) (the kernel checks every length against
  // max_seqlen before it runs)
  constexpr int64_t kPairRows = h3::kQTiles * h3::kBM;
  const int64_t pairs_by_total = (total_tokens + kPairRows - 1) / kPairRows + nseq;
  const int64_t pairs_by_max = static_cast<int64_t>(nseq) * ((max_seqlen + kPairRows - 1) / kPairRows);
  const int64_t pairs = pairs_by_total < pairs_by_max ? pairs_by_total : pairs_by_max;
  dim3 grid(static_cast<unsigned>(pairs), static_cast<unsigned>(n_heads), 1);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return head_dim == 128 ? launch_attention<128, true>(mq, mk, mv, prm, grid, s)
                         : launch_attention<64, true>(mq, mk, mv, prm, grid, s);
}

h3attn_status h3attn_qkv_fused(const void* x, const void* w, const void* bias, void* q_out, void* k_out,
                               void* v_out, int64_t n_tokens, int32_t dim_in, int32_t n_heads, int32_t head_dim,
                               int64_t x_tok_stride, const int64_t out_tok_strides[3],
                               const int64_t out_head_strides[3], const void* gamma_q, const void* gamma_k,
                               double eps, const int32_t* pos, const uint8_t* kind, int32_t sec_t, int32_t sec_h,
                               int32_t sec_w, double theta, void* stream) {
  if (!x || !w || !q_out || !k_out || !v_out) return fail(H3ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (head_dim != 64 && head_dim != 128)
    return fail(H3ATTN_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (n_tokens < 0 || n_tokens > (int64_t(1) << 31) - h3::kGemmBM)
    return fail(H3ATTN_ERR_INVALID_ARG, "n_tokens must be in [0, 2^31 - 128]");
  if (n_heads <= 0 || (static_cast<int64_t>(n_heads) * head_dim) % h3::kGemmBN != 0 ||
      static_cast<int64_t>(n_heads) * head_dim > (1 << 20))
    return fail(H3ATTN_ERR_UNSUPPORTED, "n_heads * head_dim must be a positive multiple of %d", h3::kGemmBN);
  if (dim_in <= 0 || dim_in % h3::kGemmBK != 0 || dim_in > (1 << 20))
    return fail(H3ATTN_ERR_UNSUPPORTED, "dim_in must be a positive multiple of %d", h3::kGemmBK);
  if (!aligned16(x) || !aligned16(w) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(v_out) ||
      (bias && !aligned16(bias)) || (gamma_q && !aligned16(gamma_q)) || (gamma_k && !aligned16(gamma_k)))
    return fail(H3ATTN_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  if (x_tok_stride < dim_in) return fail(H3ATTN_ERR_INVALID_ARG, "x_tok_stride must be >= dim_in");
  h3attn_status st;
  if ((st = check_strides(&x_tok_stride, 1, "x")) != H3ATTN_OK) return st;
  if ((st = check_strides(out_tok_strides, 3, "output token")) != H3ATTN_OK) return st;
  if ((st = check_strides(out_head_strides, 3, "output head")) != H3ATTN_OK) return st;
  if (!(eps >= 0.0) || !std::isfinite(eps)) return fail(H3ATTN_ERR_INVALID_ARG, "eps must be finite and >= 0");

  h3::QkvParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (pos) {
    h3::RopeTables rope;
    std::memset(&rope, 0, sizeof(rope));
    if ((st = rope_tables(&rope, kind, head_dim, sec_t, sec_h, sec_w, theta)) != H3ATTN_OK) return st;
    for (int i = 0; i < h3::kRopeMaxPairs; ++i) {  // float pairs: hi + lo = the double to ~2^-48
      prm.rope.hi3[i] = static_cast<float>(rope.inv_freq_3d[i]);
      prm.rope.lo3[i] = static_cast<float>(rope.inv_freq_3d[i] - static_cast<double>(prm.rope.hi3[i]));
      prm.rope.hi1[i] = static_cast<float>(rope.inv_freq_1d[i]);
      prm.rope.lo1[i] = static_cast<float>(rope.inv_freq_1d[i] - static_cast<double>(prm.rope.hi1[i]));
      prm.rope.axis3[i] = rope.axis_3d[i];
    }
  }
  if (n_tokens == 0) return H3ATTN_OK;
  const int64_t features = 3 * static_cast<int64_t>(n_heads) * head_dim;
  CUtensorMap mx, mw;
  if ((st = make_map_rows(&mx, x, dim_in, n_tokens, x_tok_stride, h3::kGemmBM)) != H3ATTN_OK) return st;
  if ((st = make_map_rows(&mw, w, dim_in, features, dim_in, kQkvPairs ? h3::kGemmBN / 2 : h3::kGemmBN)) !=
      H3ATTN_OK)
    return st;
  void* outs[3] = {q_out, k_out, v_out};
  // the outputs as [tokens][heads][head_dim] tensor maps with 32 x 32 boxes in the
  // 64-byte swizzle of the epilogue's staging blocks
  CUtensorMap mo[3];
  if (kQkvPairs) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(H3ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    for (int i = 0; i < 3; ++i) {
      cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(n_heads),
                            static_cast<cuuint64_t>(n_tokens)};
      cuuint64_t strides[2] = {static_cast<cuuint64_t>(out_head_strides[i]) * 2,
                               static_cast<cuuint64_t>(out_tok_strides[i]) * 2};
      cuuint32_t box[3] = {32, 1, 32};
      cuuint32_t estr[3] = {1, 1, 1};
      CUresult r = fn(&mo[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, outs[i], dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(H3ATTN_ERR_INVALID_ARG, "output tensor map rejected (%d)", (int)r);
    }
  }
  for (int i = 0; i < 3; ++i) {
    prm.out[i] = static_cast<uint16_t*>(outs[i]);
    prm.out_tok[i] = out_tok_strides[i];
    prm.out_head[i] = out_head_strides[i];
  }
  prm.bias = static_cast<const uint16_t*>(bias);
  prm.gamma[0] = static_cast<const uint16_t*>(gamma_q);
  prm.gamma[1] = static_cast<const uint16_t*>(gamma_k);
  prm.pos = pos;
  prm.kind = kind;
  prm.n_tokens = n_tokens;
  prm.dim_in = dim_in;
  prm.n_heads = n_heads;
  prm.eps = static_cast<float>(eps);
  const int tile_m = kQkvPairs ? h3::kGemmPairBM : h3::kGemmBM;
  prm.m_tiles = static_cast<int32_t>((n_tokens + tile_m - 1) / tile_m);
  prm.n_tiles = static_cast<int32_t>(features / h3::kGemmBN);
  if (static_cast<int64_t>(prm.m_tiles) * prm.n_tiles > 0x7FFFFFFF)
    return fail(H3ATTN_ERR_UNSUPPORTED, "too many tiles");
  prm.ctl.launch_id = next_launch_id();
  const int64_t tiles = static_cast<int64_t>(prm.m_tiles) * prm.n_tiles;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (kQkvPairs) {
    auto kern = head_dim == 128 ? h3::qkv_fused_pair_kernel<128> : h3::qkv_fused_pair_kernel<64>;
    e = ensure_smem_attr(kern, h3::QkvPairTraits::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(qkv pair)");
    const int pairs = resident_pairs(reinterpret_cast<const void*>(kern), h3::QkvPairTraits::kSmemBytes);
    const unsigned grid = 2u * static_cast<unsigned>(tiles < pairs ? tiles : pairs);
    kern<<<grid, h3::kGemmThreads, h3::QkvPairTraits::kSmemBytes, s>>>(mx, mw, mo[0], mo[1], mo[2], prm);
  } else {
    const unsigned grid = static_cast<unsigned>(tiles < sm_count() ? tiles : sm_count());
    auto kern = head_dim == 128 ? h3::qkv_fused_kernel<128> : h3::qkv_fused_kernel<64>;
    e = ensure_smem_attr(kern, h3::QkvTraits::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(qkv)");
    kern<<<grid, h3::kGemmThreads, h3::QkvTraits::kSmemBytes, s>>>(mx, mw, prm);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "qkv launch");
  return H3ATTN_OK;
}

}  // extern "C"
