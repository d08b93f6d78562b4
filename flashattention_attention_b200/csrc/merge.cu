// merge.cu -- combine partial attention results over disjoint key sets.
//
// A partial result over keys K_a is its normalised output o_a and the
// log-sum-exp lse_a of its scaled scores; the result over K_a and K_b is
//   lse = log(e^lse_a + e^lse_b),  o = o_a e^(lse_a - lse) + o_b e^(lse_b - lse)
// (the (m, l, O) merge of the online softmax -- kernbench2 commit, ADR-0060:
// per-step (m, l, O) state and its reduction -- written with lse = m + log l).
// The accumulator is fp32; a partial may be bf16 or fp32.  An empty key set
// has lse = -inf and weighs nothing; two empty ones stay empty.  The last
// merge can also write the final output (epilogue, output dtype).
#include "internal.h"

namespace fa {
namespace {

constexpr int kWarpsPerCta = 8;

template <typename TP, typename TO, int kPer>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc, const TP* __restrict__ o_part,
                 const float* __restrict__ lse_part, int64_t rows, int d, TO* __restrict__ out, Epilogue epi) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (row >= rows) return;
  float* acc = o_acc + row * d;
  float ca = 1.f, cb = 0.f;
  if (o_part != nullptr) {
    const float la = lse_acc[row], lb = lse_part[row];
    const float m = fmaxf(la, lb);
    if (m != -INFINITY) {
      const float wa = expf(la - m), wb = expf(lb - m), sum = wa + wb;
      ca = wa / sum;
      cb = wb / sum;
      if (lane == 0) lse_acc[row] = m + logf(sum);
    }
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int c = lane + 32 * k;
    if (c < d) {
      float o = acc[c];
      if (o_part != nullptr && cb != 0.f) o = o * ca + static_cast<float>(o_part[row * d + c]) * cb;
      if (o_part != nullptr) acc[c] = o;
      if (out != nullptr) out[row * d + c] = static_cast<TO>(apply_epilogue(o, epi));
    }
  }
}

template <typename TP, typename TO>
fa_status launch_typed(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, int64_t rows, int d,
                       void* out, const Epilogue& epi, const LaunchCtx& ctx) {
  const int64_t blocks = (rows + kWarpsPerCta - 1) / kWarpsPerCta;
  if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  auto go = [&](auto kern) {
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, ctx.stream>>>(
        o_acc, lse_acc, static_cast<const TP*>(o_part), lse_part, rows, d, static_cast<TO*>(out), epi);
    return cuda_status(cudaGetLastError());
  };
  if (d <= 64) return go(merge_kernel<TP, TO, 2>);
  if (d <= 128) return go(merge_kernel<TP, TO, 4>);
  return go(merge_kernel<TP, TO, 8>);
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
