// quant.cu -- per-row int8 KV quantiser (fkl_python PR #6, Summary,
// "compress_kv(): GPU-side per-token int8 quantization (one fp32 scale/token)").
//
// One warp per row.  Each lane holds 4 consecutive elements per 128-element
// chunk (8-byte bf16 / 16-byte fp32 vector loads, fully coalesced), the warp
// reduces max|x| with xor-shuffles, every lane divides by s = amax / 127 with
// IEEE round-to-nearest division and rounds half to even, and stores its 4
// codes as one packed 32-bit word.  Each warp handles several rows so that
// enough loads are in flight to stream HBM.
#include "internal.h"

namespace fa {
namespace {

template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
  __device__ __forceinline__ static void load(const float* p, float (&v)[4]) {
    float4 t = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  }
};
template <>
struct Vec4<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[4]) {
    uint2 t = __ldcs(reinterpret_cast<const uint2*>(p));
    // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xffff0000u);
  }
};

__device__ __forceinline__ uint32_t quantise4(const float (&v)[4], float s) {
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int c = 0;
    if (s > 0.0f) {
      c = __float2int_rn(__fdiv_rn(v[e], s));  // IEEE division, round half to even
      c = max(-127, min(127, c));
    }
    packed |= (static_cast<uint32_t>(c) & 0xffu) << (8 * e);
  }
  return packed;
}

constexpr int kWarpsPerCta = 8;

// kChunks = ceil(d / 128); kRows rows per warp.
template <typename T, int kChunks, int kRows>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    compress_kernel(const T* __restrict__ x, int64_t rows, int d, int8_t* __restrict__ codes,
                    float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t row0 = warp * kRows;
  if (row0 >= rows) return;

  float v[kRows][kChunks][4];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int col = c * 128 + lane * 4;
      const int64_t row = row0 + r;
      if (row < rows && col < d) {
        Vec4<T>::load(x + row * d + col, v[r][c]);
      } else {
        v[r][c][0] = v[r][c][1] = v[r][c][2] = v[r][c][3] = 0.0f;
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int64_t row = row0 + r;
    if (row >= rows) break;
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[r][c][e]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 127.0f);
    if (lane == 0) scales[row] = s;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int col = c * 128 + lane * 4;
      if (col < d) {
        __stcs(reinterpret_cast<unsigned int*>(codes + row * d + col), quantise4(v[r][c], s));
      }
    }
  }
}

template <typename T, int kChunks, int kRows>
fa_status launch_typed(const void* x, int64_t rows, int d, int8_t* codes, float* scales,
                       const LaunchCtx& ctx) {
  const int64_t warps = (rows + kRows - 1) / kRows;
  const int64_t blocks = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  auto kern = compress_kernel<T, kChunks, kRows>;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, ctx.stream>>>(static_cast<const T*>(x), rows,
                                                                            d, codes, scales);
  return cuda_status(cudaGetLastError());
}

template <typename T>
fa_status launch_dtype(const void* x, int64_t rows, int d, int8_t* codes, float* scales,
                       const LaunchCtx& ctx) {
  if (d <= 128) return launch_typed<T, 1, 4>(x, rows, d, codes, scales, ctx);
  if (d <= 256) return launch_typed<T, 2, 2>(x, rows, d, codes, scales, ctx);
  if (d <= 512) return launch_typed<T, 4, 1>(x, rows, d, codes, scales, ctx);
  return launch_typed<T, 8, 1>(x, rows, d, codes, scales, ctx);
}

}  // namespace

fa_status launch_compress(const void* x, int x_dtype, int64_t rows, int d, int8_t* codes, float* scales,
                          const LaunchCtx& ctx) {
  if (rows == 0) return FA_OK;
  if (x_dtype == FA_BF16) return launch_dtype<__nv_bfloat16>(x, rows, d, codes, scales, ctx);
  return launch_dtype<float>(x, rows, d, codes, scales, ctx);
}

}  // namespace fa
