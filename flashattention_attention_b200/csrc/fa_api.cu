// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// checks, dispatch to the kernels, the per-device status word, TMA
// descriptor encoding, and the watchdog self-test kernel.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <set>

#include "internal.h"

namespace fa {
namespace {

std::mutex g_mu;
constexpr int kMaxDevices = 64;
unsigned int* g_status[kMaxDevices] = {};
long long g_budget = 0;
std::set<const void*>* g_variants = nullptr;
std::atomic<long long> g_launches{0};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

long long watchdog_budget() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_budget == 0) {
    const char* e = std::getenv("FA_WATCHDOG_CYCLES");
    long long v = e ? std::atoll(e) : 0;
    g_budget = v > 0 ? v : 4000000000LL;  // about 2 s at the boost clock
  }
  return g_budget;
}

}  // namespace

// SMs of the current device (cached per device; 148 if the query fails).
int device_sm_count() {
  static std::mutex mu;
  static int counts[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

namespace {

fa_status status_word(unsigned int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status[dev] == nullptr) {
    unsigned int* p = nullptr;
    if (cudaMalloc(&p, 16) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemset(p, 0, 16) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(p);
      return FA_ERR_CUDA;
    }
    g_status[dev] = p;
  }
  *out = g_status[dev];
  return FA_OK;
}

fa_status make_ctx(fa_stream_t s, LaunchCtx* ctx) {
  ctx->stream = reinterpret_cast<cudaStream_t>(s);
  ctx->wd.budget = watchdog_budget();
  return status_word(&ctx->wd.word);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Head sizes of the tensor-core prefill: 32, 64, 96 or 128 (bf16 or int8 K/V);
// 160, 192, 224 or 256 (bf16 K/V).
bool tc_head_dim_ok(int d, int /*kv_dtype*/) {
  return d == 32 || d == 64 || d == 96 || d == 128 || d == 160 || d == 192 || d == 224 || d == 256;
}

bool epilogue_ok(const fa_epi_op* ops, int n) {
  if (n < 0 || n > FA_MAX_EPILOGUE) return false;
  for (int i = 0; i < n; ++i) {
    if (ops[i].op != FA_EPI_MUL && ops[i].op != FA_EPI_ADD) return false;
  }
  return true;
}

__global__ void watchdog_selftest_kernel(Watchdog wd) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);  // expects one arrival that never comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_parity(&bar, 0, wd, &abort_flag);
  __syncthreads();
}

}  // namespace

Epilogue make_epilogue(const fa_epi_op* ops, int n) {
  Epilogue e;
  e.n = n;
  for (int i = 0; i < 8; ++i) {
    e.op[i] = i < n ? ops[i].op : 0;
    e.val[i] = i < n ? ops[i].value : 0.f;
  }
  return e;
}

void note_variant(const void* kernel_fn) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_variants == nullptr) g_variants = new std::set<const void*>();
  g_variants->insert(kernel_fn);
}

fa_status encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                            const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                            CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  CUresult r = g_encode(map, dtype, rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported combination";
    case FA_ERR_CUDA: return "CUDA call failed";
    case FA_ERR_TIMEOUT: return "bounded device wait timed out";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

fa_status fa_compress_kv(const void* x, fa_dtype x_dtype, int64_t rows, int32_t d, int8_t* codes, float* scales,
                         fa_stream_t stream) {
  if (rows < 0 || d < 16 || d > 1024 || d % 16 != 0) return FA_ERR_INVALID;
  if (x_dtype != FA_BF16 && x_dtype != FA_F32) return FA_ERR_INVALID;
  if (rows == 0) return FA_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return FA_ERR_INVALID;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return FA_ERR_INVALID;
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_compress(x, x_dtype, rows, d, codes, scales, ctx);
}

namespace {
// Host checks of fa_attention_fwd's parameters; *launch is false when the
// call has nothing to do.  need_out = false lets out be NULL.
fa_status fwd_args(const fa_fwd_params* p, bool* launch, bool need_out = true) {
  *launch = false;
  if (p == nullptr) return FA_ERR_INVALID;
  if (p->batch < 0 || p->hq <= 0 || p->hkv <= 0 || p->hq % p->hkv != 0) return FA_ERR_INVALID;
  if (!epilogue_ok(p->epilogue, p->n_epilogue)) return FA_ERR_INVALID;
  if (!std::isfinite(p->softmax_scale)) return FA_ERR_INVALID;
  const bool varlen = p->cu_seqlens_q != nullptr;
  // with no key anywhere K, V and their scales are never read and may be NULL
  const bool no_keys = varlen ? (p->cu_seqlens_k != nullptr && p->total_k == 0) : p->seqlen_k == 0;
  if (varlen) {
    if (p->total_q < 0 || p->total_k < 0 || p->max_seqlen_q < 0 || p->max_seqlen_k < 0) return FA_ERR_INVALID;
  } else {
    if (p->seqlen_q < 0 || p->seqlen_k < 0) return FA_ERR_INVALID;
    if (p->cu_seqlens_k != nullptr) return FA_ERR_INVALID;
  }
  if (p->q_dtype == FA_F32) {
    if (p->kv_dtype != FA_F32 && p->kv_dtype != FA_I8) return FA_ERR_INVALID;
    if (p->kv_dtype == FA_I8 && !no_keys && (p->k_scales == nullptr || p->v_scales == nullptr))
      return FA_ERR_INVALID;
    if (p->head_dim <= 0 || p->head_dim % 32 != 0) return FA_ERR_INVALID;
    if (p->head_dim > 256) return FA_ERR_UNSUPPORTED;
  } else if (p->q_dtype == FA_BF16) {
    if (p->kv_dtype != FA_BF16 && p->kv_dtype != FA_I8) return FA_ERR_INVALID;
    if (p->head_dim <= 0 || p->head_dim % 32 != 0) return FA_ERR_INVALID;
    if (p->kv_dtype == FA_I8 && !no_keys && (p->k_scales == nullptr || p->v_scales == nullptr))
      return FA_ERR_INVALID;
    if (p->kv_dtype == FA_I8 && (!aligned16(p->k_scales) || !aligned16(p->v_scales))) return FA_ERR_INVALID;
    if (!tc_head_dim_ok(p->head_dim, p->kv_dtype)) return FA_ERR_UNSUPPORTED;
  } else {
    return FA_ERR_INVALID;
  }
  const bool empty = p->batch == 0 || (varlen ? p->total_q == 0 : p->seqlen_q == 0);
  if (empty) return FA_OK;
  if (p->q == nullptr || (!no_keys && (p->k == nullptr || p->v == nullptr)) || (need_out && p->out == nullptr))
    return FA_ERR_INVALID;
  if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v) || (p->out != nullptr && !aligned16(p->out)))
    return FA_ERR_INVALID;
  *launch = true;
  return FA_OK;
}
}  // namespace

fa_status fa_attention_fwd(const fa_fwd_params* p, fa_stream_t stream) {
  bool launch = false;
  fa_status st = fwd_args(p, &launch);
  if (st != FA_OK || !launch) return st;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  st = (p->q_dtype == FA_F32) ? launch_attn_f32(*p, ctx) : launch_prefill_tc(*p, nullptr, RowSink{}, ctx);
  if (st != FA_OK) return st;
  return launch_empty_rows(*p, nullptr, RowSink{}, ctx);
}

fa_status fa_attention_fwd_lse(const fa_fwd_params* p, float* lse, fa_stream_t stream) {
  bool launch = false;
  fa_status st = fwd_args(p, &launch);
  if (st != FA_OK) return st;
  if (p->q_dtype != FA_BF16) return FA_ERR_UNSUPPORTED;  // the fp32 path has no lse output
  if (!launch) return FA_OK;
  if (lse == nullptr || !aligned16(lse)) return FA_ERR_INVALID;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  RowSink sink;
  sink.lse = lse;
  st = launch_prefill_tc(*p, nullptr, sink, ctx);
  if (st != FA_OK) return st;
  return launch_empty_rows(*p, nullptr, sink, ctx);
}

fa_status fa_attention_fwd_acc(const fa_fwd_params* p, float* o_acc, float* lse_acc, int32_t flags,
                               fa_stream_t stream) {
  if ((flags & ~(FA_ACC_FIRST | FA_ACC_LAST)) != 0) return FA_ERR_INVALID;
  const bool last = (flags & FA_ACC_LAST) != 0;
  bool launch = false;
  fa_status st = fwd_args(p, &launch, last);
  if (st != FA_OK) return st;
  if (p->q_dtype != FA_BF16) return FA_ERR_UNSUPPORTED;  // the tensor-core path only
  if (!launch) return FA_OK;
  if (o_acc == nullptr || lse_acc == nullptr || !aligned16(o_acc) || !aligned16(lse_acc)) return FA_ERR_INVALID;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  RowSink sink;
  sink.acc_o = o_acc;
  sink.acc_lse = lse_acc;
  sink.first = (flags & FA_ACC_FIRST) != 0;
  sink.last = last;
  fa_fwd_params q = *p;
  if (!last) q.out = nullptr;  // not written
  st = launch_prefill_tc(q, nullptr, sink, ctx);
  if (st != FA_OK) return st;
  return launch_empty_rows(q, nullptr, sink, ctx);
}

fa_status fa_attention_merge(const fa_merge_params* p, fa_stream_t stream) {
  if (p == nullptr || p->rows < 0) return FA_ERR_INVALID;
  if (p->head_dim < 32 || p->head_dim > 256 || p->head_dim % 32 != 0) return FA_ERR_INVALID;
  if (!epilogue_ok(p->epilogue, p->n_epilogue)) return FA_ERR_INVALID;
  if (p->o_part != nullptr && p->part_dtype != FA_BF16 && p->part_dtype != FA_F32) return FA_ERR_INVALID;
  if (p->out != nullptr && p->out_dtype != FA_BF16 && p->out_dtype != FA_F32) return FA_ERR_INVALID;
  if (p->rows == 0) return FA_OK;
  if (p->o_acc == nullptr || p->lse_acc == nullptr || (p->o_part != nullptr && p->lse_part == nullptr))
    return FA_ERR_INVALID;
  if (!aligned16(p->o_acc) || !aligned16(p->lse_acc) || (p->o_part && !aligned16(p->o_part)) ||
      (p->lse_part && !aligned16(p->lse_part)) || (p->out && !aligned16(p->out)))
    return FA_ERR_INVALID;
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_merge(p->o_acc, p->lse_acc, p->o_part, p->part_dtype, p->lse_part, p->rows, p->head_dim, p->out,
                      p->out_dtype, p->epilogue, p->n_epilogue, ctx);
}

fa_status fa_attention_fwd_paged(const fa_fwd_params* p, const fa_kv_pages* pages, fa_stream_t stream) {
  if (p == nullptr || pages == nullptr) return FA_ERR_INVALID;
  if (p->batch < 0 || p->hq <= 0 || p->hkv <= 0 || p->hq % p->hkv != 0) return FA_ERR_INVALID;
  if (!epilogue_ok(p->epilogue, p->n_epilogue)) return FA_ERR_INVALID;
  if (!std::isfinite(p->softmax_scale)) return FA_ERR_INVALID;
  if (p->q_dtype != FA_BF16 || (p->kv_dtype != FA_BF16 && p->kv_dtype != FA_I8)) return FA_ERR_INVALID;
  if (p->head_dim <= 0 || p->head_dim % 32 != 0) return FA_ERR_INVALID;
  if (!tc_head_dim_ok(p->head_dim, p->kv_dtype)) return FA_ERR_UNSUPPORTED;
  if (p->kv_dtype == FA_I8 && (p->k_scales == nullptr || p->v_scales == nullptr || !aligned16(p->k_scales) ||
                               !aligned16(p->v_scales)))
    return FA_ERR_INVALID;
  if (pages->max_pages < 1 || pages->num_pages < 1 || pages->page_size < 128 || pages->page_size % 128 != 0)
    return FA_ERR_INVALID;
  if (static_cast<int64_t>(pages->num_pages) * p->hkv >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  const bool varlen = p->cu_seqlens_q != nullptr;
  if (varlen ? (p->total_q < 0 || p->max_seqlen_q < 0) : p->seqlen_q < 0) return FA_ERR_INVALID;
  const bool empty = p->batch == 0 || (varlen ? p->total_q == 0 : p->seqlen_q == 0);
  if (empty) return FA_OK;
  if (p->q == nullptr || p->k == nullptr || p->v == nullptr || p->out == nullptr || p->cu_seqlens_k == nullptr ||
      pages->block_table == nullptr)
    return FA_ERR_INVALID;
  if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v) || !aligned16(p->out) ||
      !aligned16(pages->block_table))
    return FA_ERR_INVALID;
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  st = launch_prefill_tc(*p, pages, RowSink{}, ctx);
  if (st != FA_OK) return st;
  return launch_empty_rows(*p, pages, RowSink{}, ctx);
}

size_t fa_decode_workspace_size(int32_t batch, int32_t hq, int32_t capacity, int32_t head_dim) {
  if (batch <= 0 || hq <= 0 || capacity <= 0 || head_dim <= 0) return 0;
  return decode_workspace_bytes(batch, hq, head_dim);
}

namespace {
// Host checks shared by the decode entry points (everything but the
// workspace); FA_OK means launchable, or a no-op when batch == 0.
fa_status decode_args(const fa_decode_params* p) {
  if (p == nullptr) return FA_ERR_INVALID;
  if (p->batch < 0 || p->hq <= 0 || p->hkv <= 0 || p->hq % p->hkv != 0) return FA_ERR_INVALID;
  if (p->capacity <= 0 || p->capacity % 32 != 0) return FA_ERR_INVALID;
  if (p->max_seqlen < 0 || p->max_seqlen > p->capacity) return FA_ERR_INVALID;
  if (p->split_keys < 0 || p->split_keys % 256 != 0) return FA_ERR_INVALID;
  if (!epilogue_ok(p->epilogue, p->n_epilogue)) return FA_ERR_INVALID;
  if (!std::isfinite(p->softmax_scale)) return FA_ERR_INVALID;
  if (p->kv_dtype != FA_I8 && p->kv_dtype != FA_BF16) return FA_ERR_INVALID;
  if (p->head_dim <= 0 || p->head_dim % 32 != 0) return FA_ERR_INVALID;
  // int8 or bf16 cache: 32, 64, 96, 128, 256
  if (!(p->head_dim == 32 || p->head_dim == 64 || p->head_dim == 96 || p->head_dim == 128 || p->head_dim == 256))
    return FA_ERR_UNSUPPORTED;
  if (p->batch == 0) return FA_OK;
  if (p->q == nullptr || p->k_cache == nullptr || p->v_cache == nullptr || p->out == nullptr ||
      p->cache_seqlens == nullptr)
    return FA_ERR_INVALID;
  if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->out))
    return FA_ERR_INVALID;
  if (p->kv_dtype == FA_I8) {
    if (p->k_scales == nullptr || p->v_scales == nullptr) return FA_ERR_INVALID;
    if (!aligned16(p->k_scales) || !aligned16(p->v_scales)) return FA_ERR_INVALID;
  }
  return FA_OK;
}
}  // namespace

fa_status fa_attention_decode(const fa_decode_params* p, fa_stream_t stream) {
  fa_status st = decode_args(p);
  if (st != FA_OK || p->batch == 0) return st;
  const size_t need = fa_decode_workspace_size(p->batch, p->hq, p->capacity, p->head_dim);
  if (p->workspace == nullptr || p->workspace_bytes < need || !aligned16(p->workspace)) return FA_ERR_WORKSPACE;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_decode(*p, nullptr, p->split_keys, ctx);
}

fa_status fa_attention_decode_paged(const fa_decode_params* p, const fa_kv_pages* pages, fa_stream_t stream) {
  fa_status st = decode_args(p);
  if (st != FA_OK) return st;
  if (pages == nullptr || pages->max_pages < 1 || pages->num_pages < 1 || pages->page_size < 32 ||
      pages->page_size % 32 != 0)
    return FA_ERR_INVALID;
  if (static_cast<int64_t>(pages->max_pages) * pages->page_size != p->capacity) return FA_ERR_INVALID;
  if (static_cast<int64_t>(pages->num_pages) * p->hkv * pages->page_size >= (int64_t(1) << 31))
    return FA_ERR_UNSUPPORTED;
  if (p->batch == 0) return FA_OK;
  if (pages->block_table == nullptr || !aligned16(pages->block_table)) return FA_ERR_INVALID;
  const size_t need = fa_decode_workspace_size(p->batch, p->hq, p->capacity, p->head_dim);
  if (p->workspace == nullptr || p->workspace_bytes < need || !aligned16(p->workspace)) return FA_ERR_WORKSPACE;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_decode(*p, pages, p->split_keys, ctx);
}

fa_status fa_attention_decode_noalloc(const fa_decode_params* p, fa_stream_t stream) {
  fa_status st = decode_args(p);
  if (st != FA_OK) return st;
  if (p->kv_dtype != FA_I8) return FA_ERR_UNSUPPORTED;
  if (p->batch == 0) return FA_OK;
  if (decode_noalloc_workers(p->batch, p->hq, p->hkv, p->head_dim) < 4) return FA_ERR_WORKSPACE;
  return launch_decode_noalloc(*p, p->split_keys, watchdog_budget(), reinterpret_cast<cudaStream_t>(stream));
}

namespace {
fa_status kv_append_args(const fa_kv_append_params* p) {
  if (p == nullptr) return FA_ERR_INVALID;
  if (p->batch < 0 || p->hkv < 1 || p->capacity < 1) return FA_ERR_INVALID;
  if (p->head_dim < 16 || p->head_dim > 1024 || p->head_dim % 16 != 0) return FA_ERR_INVALID;
  if (p->x_dtype != FA_BF16 && p->x_dtype != FA_F32) return FA_ERR_INVALID;
  if (p->cache_dtype != FA_I8 && p->cache_dtype != FA_BF16) return FA_ERR_INVALID;
  if (static_cast<int64_t>(p->batch) * p->hkv == 0) return FA_OK;
  if (p->k_new == nullptr || p->v_new == nullptr || p->k_cache == nullptr || p->v_cache == nullptr ||
      p->cur_pos == nullptr)
    return FA_ERR_INVALID;
  if (!aligned16(p->k_new) || !aligned16(p->v_new) || !aligned16(p->k_cache) || !aligned16(p->v_cache) ||
      !aligned16(p->cur_pos) || (p->cache_seqlens != nullptr && !aligned16(p->cache_seqlens)))
    return FA_ERR_INVALID;
  if (p->cache_dtype == FA_I8 &&
      (p->k_scales == nullptr || p->v_scales == nullptr || !aligned16(p->k_scales) || !aligned16(p->v_scales)))
    return FA_ERR_INVALID;
  if (p->cache_seqlens != nullptr) {
    // every warp of sequence b reads cur_pos[b] while one writes cache_seqlens[b]
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p->cur_pos), a1 = a0 + 4ull * p->batch;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(p->cache_seqlens), b1 = b0 + 4ull * p->batch;
    if (a0 < b1 && b0 < a1) return FA_ERR_INVALID;
  }
  return FA_OK;
}
}  // namespace

fa_status fa_kv_append(const fa_kv_append_params* p, fa_stream_t stream) {
  fa_status st = kv_append_args(p);
  if (st != FA_OK || static_cast<int64_t>(p->batch) * p->hkv == 0) return st;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_kv_append(*p, nullptr, ctx);
}

fa_status fa_kv_append_paged(const fa_kv_append_params* p, const fa_kv_pages* pages, fa_stream_t stream) {
  fa_status st = kv_append_args(p);
  if (st != FA_OK) return st;
  if (pages == nullptr || pages->max_pages < 1 || pages->num_pages < 1 || pages->page_size < 1)
    return FA_ERR_INVALID;
  if (static_cast<int64_t>(pages->max_pages) * pages->page_size != p->capacity) return FA_ERR_INVALID;
  if (static_cast<int64_t>(p->batch) * p->hkv == 0) return FA_OK;
  if (pages->block_table == nullptr || !aligned16(pages->block_table)) return FA_ERR_INVALID;
  LaunchCtx ctx;
  st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_kv_append(*p, pages, ctx);
}

fa_status fa_tq_codebook(int32_t head_dim, int32_t bits, float* levels) {
  if (levels == nullptr || head_dim < 4 || head_dim > (1 << 20) || head_dim % 2 != 0) return FA_ERR_INVALID;
  if (bits < 1 || bits > 8) return FA_ERR_INVALID;
  return tq_codebook_host(head_dim, bits, levels);
}

fa_status fa_tq_compress(const fa_tq_compress_params* p, fa_stream_t stream) {
  if (p == nullptr || p->rows < 0) return FA_ERR_INVALID;
  if (p->x_dtype != FA_BF16 && p->x_dtype != FA_F32) return FA_ERR_INVALID;
  if (p->head_dim != 64 && p->head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (p->bits < 2 || p->bits > 4) return FA_ERR_UNSUPPORTED;
  if (p->rows == 0) return FA_OK;
  if (p->x == nullptr || p->signs == nullptr || p->levels == nullptr || p->codes == nullptr || p->norms == nullptr)
    return FA_ERR_INVALID;
  if (!aligned16(p->x) || !aligned16(p->signs) || !aligned16(p->levels) || !aligned16(p->codes) ||
      !aligned16(p->norms))
    return FA_ERR_INVALID;
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_tq_compress(*p, ctx);
}

size_t fa_tq_decode_workspace_size(int32_t batch, int32_t hq, int32_t head_dim, int32_t capacity) {
  if (batch <= 0 || hq <= 0 || head_dim <= 0 || capacity <= 0) return 0;
  return static_cast<size_t>(batch) * hq * tq_decode_splits(capacity) * (head_dim + 2) * sizeof(float);
}

fa_status fa_tq_attention_decode(const fa_tq_decode_params* p, fa_stream_t stream) {
  if (p == nullptr || p->batch < 0 || p->hq <= 0 || p->hkv <= 0 || p->hq % p->hkv != 0) return FA_ERR_INVALID;
  if (p->head_dim != 64 && p->head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (p->k_bits < 2 || p->k_bits > 4 || p->v_bits < 2 || p->v_bits > 4) return FA_ERR_UNSUPPORTED;
  const int group = p->hq / p->hkv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return FA_ERR_UNSUPPORTED;
  if (p->capacity < 1 || !std::isfinite(p->softmax_scale)) return FA_ERR_INVALID;
  if (!epilogue_ok(p->epilogue, p->n_epilogue)) return FA_ERR_INVALID;
  if (p->batch == 0) return FA_OK;
  const void* ptrs[] = {p->q, p->k_codes, p->k_norms, p->v_codes, p->v_norms, p->k_levels,
                        p->v_levels, p->signs, p->cache_seqlens, p->out};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return FA_ERR_INVALID;
  const size_t need = fa_tq_decode_workspace_size(p->batch, p->hq, p->head_dim, p->capacity);
  if (p->workspace == nullptr || !aligned16(p->workspace) || p->workspace_bytes < need) return FA_ERR_WORKSPACE;
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  return launch_tq_decode(*p, static_cast<float*>(p->workspace), ctx);
}

fa_status fa_check_device_error(fa_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  // the shared word exists once some entry point has launched on this
  // device; before that there is nothing to read (and nothing is allocated)
  unsigned int* word = nullptr;
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lk(g_mu);
    word = g_status[dev];
  }
  unsigned int host = 0;
  if (word != nullptr) {
    if (cudaMemcpy(&host, word, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
    if (host != 0) {
      const unsigned int zero = 0;
      if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
    }
  }
  unsigned int noalloc = 0;
  if (take_noalloc_status(&noalloc) != FA_OK) return FA_ERR_CUDA;
  host |= noalloc;
  if (host & kStatusTimeout) return FA_ERR_TIMEOUT;
  if (host & kStatusRange) return FA_ERR_INVALID;
  return FA_OK;
}

fa_status fa_selftest_watchdog(uint64_t budget_cycles, fa_stream_t stream) {
  LaunchCtx ctx;
  fa_status st = make_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  unsigned long long b = budget_cycles;
  if (b < 1000ULL) b = 1000ULL;
  if (b > 1000000000ULL) b = 1000000000ULL;
  return launch_watchdog_selftest(b, ctx);
}

int64_t fa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t fa_kernel_variants_used(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_variants ? static_cast<int32_t>(g_variants->size()) : 0;
}

}  // extern "C"

namespace fa {
fa_status launch_watchdog_selftest(unsigned long long budget, const LaunchCtx& ctx) {
  Watchdog wd = ctx.wd;
  wd.budget = static_cast<long long>(budget);
  note_variant(reinterpret_cast<const void*>(watchdog_selftest_kernel));
  watchdog_selftest_kernel<<<1, 32, 0, ctx.stream>>>(wd);
  return cuda_status(cudaGetLastError());
}
}  // namespace fa
