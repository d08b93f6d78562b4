// merge.cu -- combine partial attention results over disjoint key sets.
//
// A partial result over keys K_a is its normalised output o_a and the
// log-sum-exp lse_a of its scaled scores; the result over K_a and K_b is
//   lse = log(e^lse_a + e^lse_b),  o = o_a e^(lse_a - lse) + o_b e^(lse_b - lse)
// (the (m, l, O) merge of the online softmax -- kernbench2 commit message,
// ADR-0060 (long context): an online-softmax merge at every ring step --
// written with lse = m + log l).  The accumulator is fp32; a partial may be
// bf16 or fp32.  An empty key set has lse = -inf and weighs nothing; two
// empty ones stay empty.  The last merge can also write the final output
// (epilogue, output dtype).
//
// HBM-bound: each thread moves four consecutive columns of one row (a float4
// of the accumulator, four elements of the partial and of the output), every
// load issued before the merge weights are known.  A CTA holds whole rows,
// so the row's lse_acc is rewritten only after all its threads have read it.
#include "internal.h"

namespace fa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                            *reinterpret_cast<const uint32_t*>(&hi));
}

template <typename TP, typename TO>
__global__ void __launch_bounds__(kThreads)
    merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc, const TP* __restrict__ o_part,
                 const float* __restrict__ lse_part, int64_t rows, int d, int rows_per_cta,
                 TO* __restrict__ out, Epilogue epi) {
  const int cpr = d / 4;  // four-column chunks per row
  const int r = threadIdx.x / cpr;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + r;
  const bool active = r < rows_per_cta && row < rows;
  const int64_t off = active ? row * d + (threadIdx.x % cpr) * 4 : 0;
  const bool merge = o_part != nullptr;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
  float la = -INFINITY, lb = -INFINITY;
  if (active) {
    a = load4(o_acc + off);
    if (merge) {
      b = load4(o_part + off);
      la = lse_acc[row];
      lb = lse_part[row];
    }
  }
  float4 y = a;
  float lse = la;
  if (merge) {
    const float m = fmaxf(la, lb);
    if (m != -INFINITY) {
      const float wa = expf(la - m), wb = expf(lb - m), sum = wa + wb;
      const float ca = wa / sum, cb = wb / sum;
      lse = m + logf(sum);
      if (cb != 0.f) {
        y = make_float4(fmaf(a.x, ca, b.x * cb), fmaf(a.y, ca, b.y * cb), fmaf(a.z, ca, b.z * cb),
                        fmaf(a.w, ca, b.w * cb));
      }
    }
    if (active) store4(o_acc + off, y);
  }
  if (out != nullptr && active) {
    store4(out + off, make_float4(apply_epilogue(y.x, epi), apply_epilogue(y.y, epi), apply_epilogue(y.z, epi),
                                  apply_epilogue(y.w, epi)));
  }
  if (merge) {
    __syncthreads();  // every thread of the row has read lse_acc[row]
    if (active && threadIdx.x % cpr == 0) lse_acc[row] = lse;
  }
}

template <typename TP, typename TO>
fa_status launch_typed(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, int64_t rows, int d,
                       void* out, const Epilogue& epi, const LaunchCtx& ctx) {
  const int rows_per_cta = kThreads / (d / 4);  // d <= 256: at least 4
  const int64_t blocks = (rows + rows_per_cta - 1) / rows_per_cta;
  if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  auto kern = merge_kernel<TP, TO>;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(blocks), kThreads, 0, ctx.stream>>>(
      o_acc, lse_acc, static_cast<const TP*>(o_part), lse_part, rows, d, rows_per_cta, static_cast<TO*>(out), epi);
  return cuda_status(cudaGetLastError());
}

}  // namespace

fa_status launch_merge(float* o_acc, float* lse_acc, const void* o_part, int part_dtype, const float* lse_part,
                       int64_t rows, int d, void* out, int out_dtype, const fa_epi_op* epi_ops, int n_epi,
                       const LaunchCtx& ctx) {
  if (rows == 0) return FA_OK;
  const Epilogue epi = make_epilogue(epi_ops, n_epi);
  const bool part_bf = part_dtype == FA_BF16, out_bf = out_dtype == FA_BF16;
  if (part_bf && out_bf) return launch_typed<__nv_bfloat16, __nv_bfloat16>(o_acc, lse_acc, o_part, lse_part, rows, d, out, epi, ctx);
  if (part_bf) return launch_typed<__nv_bfloat16, float>(o_acc, lse_acc, o_part, lse_part, rows, d, out, epi, ctx);
  if (out_bf) return launch_typed<float, __nv_bfloat16>(o_acc, lse_acc, o_part, lse_part, rows, d, out, epi, ctx);
  return launch_typed<float, float>(o_acc, lse_acc, o_part, lse_part, rows, d, out, epi, ctx);
}

}  // namespace fa
