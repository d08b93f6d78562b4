// quant.cu -- per-row int8 KV quantiser (fkl_python PR #6, Summary: the
// cache compressed on the GPU to int8 codes per token, one fp32 scale each).
//
// compress_kernel (any d): one warp per row; compress_rows8_kernel (d = 64
// and 128, further below): eight lanes per row.  In the first, each lane
// holds 4 consecutive elements per 128-element chunk (8-byte bf16 / 16-byte
// fp32 vector loads, fully coalesced), the warp reduces max|x| with
// xor-shuffles, and every lane forms c = rint(x / s) with
// s = amax / 127 (IEEE division, once per row), rounds half to even, and
// stores its 4 codes as one packed 32-bit word.  Each warp handles several
// rows so that enough loads are in flight to stream HBM.
//
// The quotient x / s must be the IEEE round-to-nearest one (the codes are
// compared bit for bit with an fp32 reference).  A full division per element
// made the kernel issue-bound, so the row computes y = RN(1 / s) once and
// every element takes Markstein's correction step (P. Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): q0 = RN(x y), e = x - q0 s (exact with an FMA),
// q = RN(q0 + e y).  With y correctly rounded and q0 within an ulp of x / s,
// q is the correctly rounded quotient as long as no intermediate leaves the
// normal range; rows with s outside [2^-60, 2^60] take the IEEE division.
// Then |q| <= amax / s < 127.5 (s = RN(amax / 127) is within 2^-24 of
// amax / 127), so no clamp is needed, and adding 1.5 * 2^23 rounds q half to
// even into the low mantissa bits, whose low byte is the two's-complement code.
#include "internal.h"

namespace fa {
namespace {

// Raw vector loads of 4 consecutive elements (kept raw in registers while
// the next rows are in flight) and their exact widening to fp32.
template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
  using Raw = float4;
  __device__ __forceinline__ static Raw load(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
  __device__ __forceinline__ static Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ static void widen(const Raw& t, float (&v)[4]) {
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  }
};
template <>
struct Vec4<__nv_bfloat16> {
  using Raw = uint2;
  __device__ __forceinline__ static Raw load(const __nv_bfloat16* p) {
    return __ldcs(reinterpret_cast<const uint2*>(p));
  }
  __device__ __forceinline__ static Raw zero() { return make_uint2(0u, 0u); }
  // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
  __device__ __forceinline__ static void widen(const Raw& t, float (&v)[4]) {
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xffff0000u);
  }
};

// IEEE-division path: any s (0 gives zero codes), with the clamp.
__device__ __forceinline__ uint32_t quantise4_div(const float (&v)[4], float s) {
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

// Fast path for s in [2^-60, 2^60]: y = RN(1 / s); Markstein's correction
// step gives the correctly rounded x / s, and the 1.5 * 2^23 shift rounds it
// half to even into the low byte.
__device__ __forceinline__ uint32_t quantise4_fast(const float (&v)[4], float s, float y) {
  const float2 y2 = make_float2(y, y), ns2 = make_float2(-s, -s);
  const float2 shift = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  uint32_t t[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float2 x = make_float2(v[2 * h], v[2 * h + 1]);
    const float2 q0 = mul2(x, y2);
    const float2 r = fma2(q0, ns2, x);  // x - q0 s, exact
    const float2 q = fma2(r, y2, q0);
    const float2 k = add2(q, shift);
    t[2 * h] = __float_as_uint(k.x);
    t[2 * h + 1] = __float_as_uint(k.y);
  }
  uint32_t lo, hi, packed;
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(t[0]), "r"(t[1]));
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(t[2]), "r"(t[3]));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(packed) : "r"(lo), "r"(hi));
  return packed;
}

constexpr int kWarpsPerCta = 8;

// kChunks = ceil(d / 128); a warp quantises groups of kRows rows, striding
// over the groups of a persistent grid, with the next group's loads in
// flight while it works on the current one.
template <typename T, int kChunks, int kRows>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    compress_kernel(const T* __restrict__ x, int64_t rows, int d, int8_t* __restrict__ codes,
                    float* __restrict__ scales) {
  using V = Vec4<T>;
  using Raw = typename V::Raw;
  const int lane = threadIdx.x & 31;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
  const int64_t n_groups = (rows + kRows - 1) / kRows;
  int64_t g = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (g >= n_groups) return;

  auto load = [&](int64_t grp, Raw (&buf)[kRows][kChunks]) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int col = c * 128 + lane * 4;
        const int64_t row = grp * kRows + r;
        buf[r][c] = (row < rows && col < d) ? V::load(x + row * d + col) : V::zero();
      }
    }
  };
  Raw cur[kRows][kChunks], nxt[kRows][kChunks];
  load(g, cur);
  for (; g < n_groups; g += n_warps) {
    if (g + n_warps < n_groups) load(g + n_warps, nxt);
    float s_own = 0.f;  // lane r < kRows keeps row r's scale for one combined store
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t row = g * kRows + r;
      float v[kChunks][4];
      float amax = 0.0f;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        V::widen(cur[r][c], v[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float s = __fdiv_rn(amax, 127.0f);
      if (lane == r) s_own = s;
      const bool fast = s >= 0x1p-60f && s <= 0x1p60f;  // warp-uniform
      const float y = fast ? __frcp_rn(s) : 0.0f;
      if (row < rows) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int col = c * 128 + lane * 4;
          if (col < d) {
            const uint32_t packed = fast ? quantise4_fast(v[c], s, y) : quantise4_div(v[c], s);
            __stcs(reinterpret_cast<unsigned int*>(codes + row * d + col), packed);
          }
        }
      }
    }
    if (lane < kRows && g * kRows + lane < rows) scales[g * kRows + lane] = s_own;
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int c = 0; c < kChunks; ++c) cur[r][c] = nxt[r][c];
  }
}

// d = 8 kE (64 or 128): eight lanes per row, kE consecutive elements per
// lane in 16-byte loads, four rows per warp pass, so each row's max|x| takes
// three shuffles and one warp instruction forms four rows' scales and
// reciprocals.  Persistent grid with the next pass's loads in flight; codes
// leave as one 8- or 16-byte store per lane, the four scales as one 16-byte
// span.
template <typename T, int kE>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    compress_rows8_kernel(const T* __restrict__ x, int64_t rows, int8_t* __restrict__ codes,
                          float* __restrict__ scales) {
  constexpr int kD = 8 * kE;
  constexpr int kVec = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte load
  constexpr int kLoads = kE / kVec;
  const int lane = threadIdx.x & 31, sub = lane & 7, grp = lane >> 3;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
  const int64_t n_pass = (rows + 3) / 4;
  int64_t g = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (g >= n_pass) return;
  auto load = [&](int64_t pass, uint4 (&buf)[kLoads]) {
    const int64_t row = pass * 4 + grp;
#pragma unroll
    for (int i = 0; i < kLoads; ++i)
      buf[i] = row < rows ? __ldcs(reinterpret_cast<const uint4*>(x + row * kD + sub * kE + i * kVec))
                          : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 cur[kLoads], nxt[kLoads];
  load(g, cur);
  for (; g < n_pass; g += n_warps) {
    if (g + n_warps < n_pass) load(g + n_warps, nxt);
    float v[kE];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      const uint32_t w[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if constexpr (sizeof(T) == 2) {
          // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits
          v[i * kVec + 2 * j] = __uint_as_float(w[j] << 16);
          v[i * kVec + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        } else {
          v[i * kVec + j] = __uint_as_float(w[j]);
        }
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < kE; ++e) amax = fmaxf(amax, fabsf(v[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float s = __fdiv_rn(amax, 127.0f);
    const bool fast = s >= 0x1p-60f && s <= 0x1p60f;  // uniform over the row's 8 lanes
    const float y = fast ? __frcp_rn(s) : 0.0f;
    uint32_t packed[kE / 4];
#pragma unroll
    for (int q = 0; q < kE / 4; ++q) {
      const float v4[4] = {v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]};
      packed[q] = fast ? quantise4_fast(v4, s, y) : quantise4_div(v4, s);
    }
    const int64_t row = g * 4 + grp;
    if (row < rows) {
      int8_t* dst = codes + row * kD + sub * kE;
      if constexpr (kE == 16) {
        __stcs(reinterpret_cast<uint4*>(dst), make_uint4(packed[0], packed[1], packed[2], packed[3]));
      } else {
        __stcs(reinterpret_cast<uint2*>(dst), make_uint2(packed[0], packed[1]));
      }
      if (sub == 0) scales[row] = s;
    }
#pragma unroll
    for (int i = 0; i < kLoads; ++i) cur[i] = nxt[i];
  }
}

template <typename T, int kE>
fa_status launch_rows8(const void* x, int64_t rows, int8_t* codes, float* scales, const LaunchCtx& ctx) {
  const int64_t passes = (rows + 3) / 4;
  int64_t blocks = (passes + kWarpsPerCta - 1) / kWarpsPerCta;
  auto kern = compress_rows8_kernel<T, kE>;
  static int per_sm = 0;  // resident CTAs per SM (register-limited), queried once
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kWarpsPerCta * 32, 0) != cudaSuccess || n <= 0)
      return FA_ERR_CUDA;
    per_sm = n;
  }
  const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
  if (blocks > resident) blocks = resident;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, ctx.stream>>>(static_cast<const T*>(x), rows, codes,
                                                                            scales);
  return cuda_status(cudaGetLastError());
}

template <typename T, int kChunks, int kRows>
fa_status launch_typed(const void* x, int64_t rows, int d, int8_t* codes, float* scales,
                       const LaunchCtx& ctx) {
  const int64_t groups = (rows + kRows - 1) / kRows;
  int64_t blocks = (groups + kWarpsPerCta - 1) / kWarpsPerCta;
  auto kern = compress_kernel<T, kChunks, kRows>;
  static int per_sm = 0;  // resident CTAs per SM (register-limited), queried once
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kWarpsPerCta * 32, 0) != cudaSuccess || n <= 0)
      return FA_ERR_CUDA;
    per_sm = n;
  }
  const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
  if (blocks > resident) blocks = resident;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, ctx.stream>>>(static_cast<const T*>(x), rows,
                                                                            d, codes, scales);
  return cuda_status(cudaGetLastError());
}

template <typename T>
fa_status launch_dtype(const void* x, int64_t rows, int d, int8_t* codes, float* scales,
                       const LaunchCtx& ctx) {
  if (d == 128) return launch_rows8<T, 16>(x, rows, codes, scales, ctx);
  if (d == 64) return launch_rows8<T, 8>(x, rows, codes, scales, ctx);
  if (d <= 128) return launch_typed<T, 1, 4>(x, rows, d, codes, scales, ctx);
  if (d <= 256) return launch_typed<T, 2, 2>(x, rows, d, codes, scales, ctx);
  if (d <= 512) return launch_typed<T, 4, 1>(x, rows, d, codes, scales, ctx);
  return launch_typed<T, 8, 1>(x, rows, d, codes, scales, ctx);
}

// ---------------------------------------------------------------- cache append
// One new token per sequence: rows u = b * hkv + g of k_new / v_new go to
// cache row u * capacity + cur_pos[b] (dense) or to token cur_pos[b] %
// page_size of page block_table[b][cur_pos[b] / page_size] (paged),
// quantised exactly as compress_kernel does, or stored as bf16.  One warp per
// (K or V, u) row; lane layout and arithmetic as in compress_kernel.  A slot
// outside [0, capacity), or a page outside the pool, is not written and is
// reported in the status word.
struct AppendArgs {
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  float* k_scales;
  float* v_scales;
  const int32_t* cur_pos;
  int32_t* seqlens;  // optional: seqlens[b] = cur_pos[b] + 1
  int batch, hkv, d, capacity, cache_i8;
  // paged caches (null table: dense): pool [num_pages, hkv, page_size, d]
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  Watchdog wd;
};

template <typename T, int kChunks>
__global__ void __launch_bounds__(kWarpsPerCta * 32) kv_append_kernel(const AppendArgs A) {
  using V = Vec4<T>;
  const int lane = threadIdx.x & 31;
  const int64_t units = static_cast<int64_t>(A.batch) * A.hkv;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (w >= 2 * units) return;
  const bool is_v = w >= units;
  const int64_t u = is_v ? w - units : w;
  const int b = static_cast<int>(u / A.hkv);
  const int pos = A.cur_pos[b];
  if (pos < 0 || pos >= A.capacity) {
    if (lane == 0) record_status(A.wd, kStatusRange);
    return;
  }
  int64_t row = u * A.capacity + pos;
  if (A.block_table != nullptr) {
    const int pg = A.block_table[static_cast<int64_t>(b) * A.max_pages + pos / A.page_size];
    if (pg < 0 || pg >= A.num_pages) {
      if (lane == 0) record_status(A.wd, kStatusRange);
      return;
    }
    row = (static_cast<int64_t>(pg) * A.hkv + (u % A.hkv)) * A.page_size + pos % A.page_size;
  }
  if (A.seqlens != nullptr && !is_v && u % A.hkv == 0 && lane == 0) A.seqlens[b] = pos + 1;
  const T* src = static_cast<const T*>(is_v ? A.v_new : A.k_new) + u * A.d;
  float v[kChunks][4];
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int col = c * 128 + lane * 4;
    if (col < A.d) {
      V::widen(V::load(src + col), v[c]);
    } else {
      v[c][0] = v[c][1] = v[c][2] = v[c][3] = 0.0f;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
  }
  if (!A.cache_i8) {
    // bf16 cache: the row as bf16 (exact for bf16 input, RNE for fp32)
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(is_v ? A.v_cache : A.k_cache) + row * A.d;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int col = c * 128 + lane * 4;
      if (col < A.d) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v[c][0], v[c][1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(v[c][2], v[c][3]);
        *reinterpret_cast<uint2*>(dst + col) =
            make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
      }
    }
    return;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = __fdiv_rn(amax, 127.0f);
  const bool fast = s >= 0x1p-60f && s <= 0x1p60f;  // warp-uniform
  const float y = fast ? __frcp_rn(s) : 0.0f;
  int8_t* codes = static_cast<int8_t*>(is_v ? A.v_cache : A.k_cache) + row * A.d;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int col = c * 128 + lane * 4;
    if (col < A.d) {
      const uint32_t packed = fast ? quantise4_fast(v[c], s, y) : quantise4_div(v[c], s);
      *reinterpret_cast<uint32_t*>(codes + col) = packed;
    }
  }
  if (lane == 0) (is_v ? A.v_scales : A.k_scales)[row] = s;
}

template <typename T, int kChunks>
fa_status launch_append_typed(const AppendArgs& A, const LaunchCtx& ctx) {
  const int64_t rows = 2LL * A.batch * A.hkv;
  const int64_t blocks = (rows + kWarpsPerCta - 1) / kWarpsPerCta;
  if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  auto kern = kv_append_kernel<T, kChunks>;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, ctx.stream>>>(A);
  return cuda_status(cudaGetLastError());
}

template <typename T>
fa_status launch_append_dtype(const AppendArgs& A, const LaunchCtx& ctx) {
  if (A.d <= 128) return launch_append_typed<T, 1>(A, ctx);
  if (A.d <= 256) return launch_append_typed<T, 2>(A, ctx);
  if (A.d <= 512) return launch_append_typed<T, 4>(A, ctx);
  return launch_append_typed<T, 8>(A, ctx);
}

}  // namespace

fa_status launch_compress(const void* x, int x_dtype, int64_t rows, int d, int8_t* codes, float* scales,
                          const LaunchCtx& ctx) {
  if (rows == 0) return FA_OK;
  if (x_dtype == FA_BF16) return launch_dtype<__nv_bfloat16>(x, rows, d, codes, scales, ctx);
  return launch_dtype<float>(x, rows, d, codes, scales, ctx);
}

}  // namespace fa

namespace fa {

fa_status launch_kv_append(const fa_kv_append_params& p, const fa_kv_pages* pages, const LaunchCtx& ctx) {
  AppendArgs A;
  A.block_table = pages != nullptr ? pages->block_table : nullptr;
  A.max_pages = pages != nullptr ? pages->max_pages : 1;
  A.page_size = pages != nullptr ? pages->page_size : p.capacity;
  A.num_pages = pages != nullptr ? pages->num_pages : p.batch;
  A.k_new = p.k_new;
  A.v_new = p.v_new;
  A.k_cache = p.k_cache;
  A.v_cache = p.v_cache;
  A.k_scales = p.k_scales;
  A.v_scales = p.v_scales;
  A.cur_pos = p.cur_pos;
  A.seqlens = p.cache_seqlens;
  A.batch = p.batch;
  A.hkv = p.hkv;
  A.d = p.head_dim;
  A.capacity = p.capacity;
  A.cache_i8 = p.cache_dtype == FA_I8 ? 1 : 0;
  A.wd = ctx.wd;
  if (static_cast<int64_t>(p.batch) * p.hkv == 0) return FA_OK;
  if (p.x_dtype == FA_BF16) return launch_append_dtype<__nv_bfloat16>(A, ctx);
  return launch_append_dtype<float>(A, ctx);
}

}  // namespace fa
