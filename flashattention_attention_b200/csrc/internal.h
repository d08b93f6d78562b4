// internal.h -- launchers shared between the C-ABI host layer (fa_api.cu) and
// the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>

#include "device.cuh"
#include "fa.h"

namespace fa {

struct LaunchCtx {
  cudaStream_t stream;
  Watchdog wd;
};

Epilogue make_epilogue(const fa_epi_op* ops, int n);

// Records that a kernel instantiation was launched (distinct-variant count).
void note_variant(const void* kernel_fn);

fa_status launch_compress(const void* x, int x_dtype, int64_t rows, int d, int8_t* codes, float* scales,
                          const LaunchCtx& ctx);
fa_status launch_kv_append(const fa_kv_append_params& p, const fa_kv_pages* pages, const LaunchCtx& ctx);
fa_status launch_attn_f32(const fa_fwd_params& p, const LaunchCtx& ctx);

// How the tensor-core prefill hands over its rows: the normalised output
// (all null), that output with its per-row log-sum-exp (lse), or merged into
// an fp32 accumulator (acc_o, acc_lse; see fa_attention_fwd_acc).
struct RowSink {
  float* lse = nullptr;
  float* acc_o = nullptr;
  float* acc_lse = nullptr;
  int first = 0;  // the accumulator holds nothing yet and is not read
  int last = 0;   // the merged rows go to out; the accumulator is left as it was
};

fa_status launch_empty_rows(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink,
                            const LaunchCtx& ctx);
fa_status launch_prefill_tc(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink,
                            const LaunchCtx& ctx);
fa_status launch_merge(float* o_acc, float* lse_acc, const void* o_part, int part_dtype, const float* lse_part,
                       int64_t rows, int d, void* out, int out_dtype, const fa_epi_op* epi, int n_epi,
                       const LaunchCtx& ctx);
fa_status launch_decode(const fa_decode_params& p, const fa_kv_pages* pages, int split_keys, const LaunchCtx& ctx);
// TurboQuant: keys per split of the decode, its split count, launchers and the host codebook
constexpr int kTqSplitKeys = 2048;
int tq_decode_splits(int capacity);
fa_status launch_tq_compress(const fa_tq_compress_params& p, const LaunchCtx& ctx);
fa_status launch_tq_decode(const fa_tq_decode_params& p, float* part, const LaunchCtx& ctx);
fa_status tq_codebook_host(int d, int bits, float* levels);
size_t decode_workspace_bytes(int batch, int hq, int head_dim);
int decode_noalloc_workers(int batch, int hq, int hkv, int head_dim);
fa_status launch_decode_noalloc(const fa_decode_params& p, int split_keys, long long budget, cudaStream_t stream);
size_t decode_noalloc_scratch_bytes();
fa_status take_noalloc_status(unsigned int* bits);
fa_status launch_watchdog_selftest(unsigned long long budget, const LaunchCtx& ctx);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
fa_status encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                            const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                            CUtensorMapSwizzle swizzle);

// SMs of the current device (cached per device).
int device_sm_count();

inline fa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

}  // namespace fa
