// attn_f32.cu -- fp32 attention on the CUDA cores, and the empty-band rows.
//
// attn_f32_kernel: the correctness tier for fp32 inputs (fkl_python PR #6,
// Verification: the dense causal check at head size 64 reaches errors near
// 1e-7, which needs fp32 products, so no TF32 tensor cores here).  Same masks, GQA, varlen and
// epilogue semantics as the tensor-core path.  A CTA owns 32 query rows of one
// (sequence, q-head); four threads share a row, each holding every 16th group
// of 4 dims, so the K/V tiles in shared memory are read without bank
// conflicts.  Keys stream in tiles of 32 through an online softmax (running
// max m and sum l in fp32, exp2 with log2(e) folded into the scale).
// With an int8 KV cache (fkl_python PR #6, Verification: int8-cache
// attention checked against an oracle on the dequantised cache) each K/V element enters the shared tile as c * s
// rounded once to fp32 (a 7-bit |c| times a 24-bit significand can need 31
// bits: relative error at most 2^-24, far inside the fp32 path's tolerance).
//
// empty_rows_kernel: rows whose band is empty (causal with s_q > s_k leaves
// rows i < s_q - s_k without keys; s_k = 0 leaves every row without keys)
// get uniform weights over all s_k keys, i.e. the mean of V, zeros for s_k =
// 0 (SKaiNET-transformers PR #419, Summary: a sliding-window row whose band
// holds no key falls back to the uniform softmax), then the epilogue.  The main
// kernels skip those rows.  Partial results (an lse output) or an
// accumulator to merge into give such rows no weight instead.
#include "internal.h"
#include "layout.cuh"

namespace fa {
namespace {

constexpr int kRowsPerCta = 32;
constexpr int kKeysPerTile = 32;
constexpr float kLog2e = 1.4426950408889634f;

// Four consecutive K or V elements of row `row` as fp32: plain fp32, or int8
// codes times the row's scale.
template <bool kI8>
__device__ __forceinline__ float4 load_kv4(const void* base, const float* scales, int64_t row, int d, int col) {
  if constexpr (kI8) {
    const char4 c = *reinterpret_cast<const char4*>(static_cast<const int8_t*>(base) + row * d + col);
    const float s = scales[row];
    return make_float4(static_cast<float>(c.x) * s, static_cast<float>(c.y) * s, static_cast<float>(c.z) * s,
                       static_cast<float>(c.w) * s);
  } else {
    return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + row * d + col);
  }
}

template <int D, bool kI8>
__global__ void __launch_bounds__(128)
    attn_f32_kernel(const float* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
                    const float* __restrict__ k_scales, const float* __restrict__ v_scales,
                    float* __restrict__ out, SeqLayout L, int hq, int hkv, float scale_log2, Epilogue epi) {
  constexpr int kPer = D / 4;        // dims per thread
  constexpr int kVec = kPer / 4;     // float4 groups per thread
  extern __shared__ __align__(16) float f32_smem[];
  float (*ks)[D] = reinterpret_cast<float (*)[D]>(f32_smem);
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(f32_smem + kKeysPerTile * D);

  const int b = blockIdx.z, h = blockIdx.y;
  const int g = h / (hq / hkv);
  const Seq sq = seq_of(L, b, h, g);
  const int row_base = blockIdx.x * kRowsPerCta;
  if (row_base >= sq.s_q) return;

  const int t = threadIdx.x;
  const int r = t >> 2, part = t & 3;
  const int i = row_base + r;
  const bool row_ok = i < sq.s_q;

  // this thread's dims: group m (0..kVec-1) covers dims 16*m + 4*part .. +3
  float qr[kPer], o[kPer];
#pragma unroll
  for (int m = 0; m < kVec; ++m) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row_ok) x = *reinterpret_cast<const float4*>(q + (sq.q_row0 + i) * D + 16 * m + 4 * part);
    qr[4 * m + 0] = x.x; qr[4 * m + 1] = x.y; qr[4 * m + 2] = x.z; qr[4 * m + 3] = x.w;
  }
#pragma unroll
  for (int c = 0; c < kPer; ++c) o[c] = 0.f;

  // key range touched by any row of this CTA
  int lo_a, hi_a, lo_b, hi_b;
  band_of(L, row_base, sq.s_q, sq.s_k, lo_a, hi_a);
  band_of(L, min(row_base + kRowsPerCta, sq.s_q) - 1, sq.s_q, sq.s_k, lo_b, hi_b);
  const int k_lo = max(0, lo_a), k_hi = min(sq.s_k, hi_b);
  int my_lo, my_hi;
  band_of(L, i, sq.s_q, sq.s_k, my_lo, my_hi);

  float m_run = -INFINITY, l_run = 0.f;
  for (int j0 = (k_lo / kKeysPerTile) * kKeysPerTile; j0 < k_hi; j0 += kKeysPerTile) {
    __syncthreads();
    for (int e = t; e < kKeysPerTile * D / 4; e += 128) {
      const int jj = e / (D / 4), c4 = e % (D / 4);
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j0 + jj < sq.s_k) {
        kv = load_kv4<kI8>(k, k_scales, sq.k_row0 + j0 + jj, D, 4 * c4);
        vv = load_kv4<kI8>(v, v_scales, sq.k_row0 + j0 + jj, D, 4 * c4);
      }
      *reinterpret_cast<float4*>(&ks[jj][4 * c4]) = kv;
      *reinterpret_cast<float4*>(&vs[jj][4 * c4]) = vv;
    }
    __syncthreads();

    float s[kKeysPerTile];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKeysPerTile; ++jj) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < kVec; ++m) {
        const float4 kv = *reinterpret_cast<const float4*>(&ks[jj][16 * m + 4 * part]);
        acc = fmaf(qr[4 * m + 0], kv.x, acc);
        acc = fmaf(qr[4 * m + 1], kv.y, acc);
        acc = fmaf(qr[4 * m + 2], kv.z, acc);
        acc = fmaf(qr[4 * m + 3], kv.w, acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      const int j = j0 + jj;
      s[jj] = (j >= my_lo && j < my_hi) ? acc * scale_log2 : -INFINITY;
      tmax = fmaxf(tmax, s[jj]);
    }
    const float m_new = fmaxf(m_run, tmax);
    const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(m_run - m_ref);
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < kPer; ++c) o[c] *= alpha;
#pragma unroll
    for (int jj = 0; jj < kKeysPerTile; ++jj) {
      const float pj = exp2f(s[jj] - m_ref);
      psum += pj;
#pragma unroll
      for (int m = 0; m < kVec; ++m) {
        const float4 vv = *reinterpret_cast<const float4*>(&vs[jj][16 * m + 4 * part]);
        o[4 * m + 0] = fmaf(pj, vv.x, o[4 * m + 0]);
        o[4 * m + 1] = fmaf(pj, vv.y, o[4 * m + 1]);
        o[4 * m + 2] = fmaf(pj, vv.z, o[4 * m + 2]);
        o[4 * m + 3] = fmaf(pj, vv.w, o[4 * m + 3]);
      }
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
  }

  if (!row_ok || my_lo >= my_hi) return;  // empty band: written by empty_rows_kernel
  const float inv_l = 1.0f / l_run;
#pragma unroll
  for (int m = 0; m < kVec; ++m) {
    float4 y;
    y.x = apply_epilogue(o[4 * m + 0] * inv_l, epi);
    y.y = apply_epilogue(o[4 * m + 1] * inv_l, epi);
    y.z = apply_epilogue(o[4 * m + 2] * inv_l, epi);
    y.w = apply_epilogue(o[4 * m + 3] * inv_l, epi);
    *reinterpret_cast<float4*>(out + (sq.q_row0 + i) * D + 16 * m + 4 * part) = y;
  }
}

// ---------------------------------------------------------------- empty band
template <typename TV, typename TO>
__global__ void __launch_bounds__(128)
    empty_rows_kernel(const TV* __restrict__ v, const float* __restrict__ v_scales, TO* __restrict__ out,
                      RowSink sink, SeqLayout L, int hq, int hkv, int d, Epilogue epi) {
  const int b = blockIdx.y, h = blockIdx.x;
  const int g = h / (hq / hkv);
  const Seq sq = seq_of(L, b, h, g);
  // rows i < n_empty have no visible key (a window never empties a row that
  // the causal mask leaves a key)
  const int n_empty = sq.s_k == 0 ? sq.s_q : (L.causal ? min(sq.s_q, sq.s_q - sq.s_k) : 0);
  if (n_empty <= 0) return;
  if (sink.acc_o != nullptr) {
    // merging nothing: the accumulator stays (or starts empty); the last
    // step writes it out
    for (int i = 0; i < n_empty; ++i) {
      const int64_t row = sq.q_row0 + i;
      for (int c = threadIdx.x; c < d; c += blockDim.x) {
        const float a = sink.first ? 0.f : sink.acc_o[row * d + c];
        if (sink.last) {
          out[row * d + c] = static_cast<TO>(apply_epilogue(a, epi));
        } else if (sink.first) {
          sink.acc_o[row * d + c] = 0.f;
        }
      }
      if (threadIdx.x == 0 && sink.first && !sink.last) sink.acc_lse[row] = -INFINITY;
    }
    return;
  }
  if (sink.lse != nullptr) {
    // partial results: rows without keys carry no weight (lse = -inf)
    const TO zero = static_cast<TO>(apply_epilogue(0.f, epi));
    for (int i = 0; i < n_empty; ++i) {
      for (int c = threadIdx.x; c < d; c += blockDim.x) out[(sq.q_row0 + i) * d + c] = zero;
      if (threadIdx.x == 0) sink.lse[sq.q_row0 + i] = -INFINITY;
    }
    return;
  }
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float sum = 0.f;
    for (int j = 0; j < sq.s_k; ++j) {
      int64_t row = sq.k_row0 + j;
      if (L.block_table != nullptr) {
        int plane, prow;
        bool bad;
        paged_key(L, b, g, j, plane, prow, bad);  // a bad page id is reported by the prefill kernel
        row = static_cast<int64_t>(plane) * L.page_size + prow;
      }
      float x;
      if constexpr (sizeof(TV) == 1) {
        x = static_cast<float>(v[row * d + c]) * v_scales[row];
      } else {
        x = static_cast<float>(v[row * d + c]);
      }
      sum += x;
    }
    const float y = apply_epilogue(sq.s_k > 0 ? sum / static_cast<float>(sq.s_k) : 0.f, epi);
    for (int i = 0; i < n_empty; ++i) out[(sq.q_row0 + i) * d + c] = static_cast<TO>(y);
  }
}

template <int D>
fa_status launch_f32_d(const fa_fwd_params& p, const LaunchCtx& ctx) {
  const SeqLayout L = SeqLayout::from(p);
  const int max_sq = p.cu_seqlens_q ? p.max_seqlen_q : p.seqlen_q;
  dim3 grid((max_sq + kRowsPerCta - 1) / kRowsPerCta, p.hq, p.batch);
  if (grid.x == 0) return FA_OK;
  auto kern = p.kv_dtype == FA_I8 ? attn_f32_kernel<D, true> : attn_f32_kernel<D, false>;
  constexpr int kSmem = 2 * kKeysPerTile * D * sizeof(float);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
    return FA_ERR_CUDA;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<grid, 128, kSmem, ctx.stream>>>(static_cast<const float*>(p.q), p.k, p.v, p.k_scales, p.v_scales,
                                     static_cast<float*>(p.out), L, p.hq, p.hkv, p.softmax_scale * kLog2e,
                                     make_epilogue(p.epilogue, p.n_epilogue));
  return cuda_status(cudaGetLastError());
}

}  // namespace

fa_status launch_attn_f32(const fa_fwd_params& p, const LaunchCtx& ctx) {
  switch (p.head_dim) {
    case 32: return launch_f32_d<32>(p, ctx);
    case 64: return launch_f32_d<64>(p, ctx);
    case 96: return launch_f32_d<96>(p, ctx);
    case 128: return launch_f32_d<128>(p, ctx);
    case 160: return launch_f32_d<160>(p, ctx);
    case 192: return launch_f32_d<192>(p, ctx);
    case 224: return launch_f32_d<224>(p, ctx);
    case 256: return launch_f32_d<256>(p, ctx);
    default: return FA_ERR_UNSUPPORTED;
  }
}

fa_status launch_empty_rows(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink,
                            const LaunchCtx& ctx) {
  // Rows lose every key only to the causal mask with s_q > s_k, or when
  // s_k = 0.  Dense inputs decide it here; varlen self-attention (one
  // cu_seqlens for both) has s_q = s_k per sequence, so the diagonal (or,
  // without the causal mask, every key) stays visible; separate varlen key
  // counts and paged keys are decided per sequence on the device.
  if (pages == nullptr) {
    if (p.cu_seqlens_q == nullptr && p.seqlen_k > 0 && (!p.causal || p.seqlen_q <= p.seqlen_k)) return FA_OK;
    if (p.cu_seqlens_q != nullptr && (p.cu_seqlens_k == nullptr || p.cu_seqlens_k == p.cu_seqlens_q))
      return FA_OK;
  }
  const SeqLayout L = pages != nullptr ? SeqLayout::paged(p, *pages) : SeqLayout::from(p);
  const Epilogue epi = make_epilogue(p.epilogue, p.n_epilogue);
  dim3 grid(p.hq, p.batch);
  if (p.q_dtype == FA_F32 && p.kv_dtype == FA_I8) {
    auto kern = empty_rows_kernel<int8_t, float>;
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<grid, 128, 0, ctx.stream>>>(static_cast<const int8_t*>(p.v), p.v_scales, static_cast<float*>(p.out),
                                       sink, L, p.hq, p.hkv, p.head_dim, epi);
  } else if (p.q_dtype == FA_F32) {
    auto kern = empty_rows_kernel<float, float>;
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<grid, 128, 0, ctx.stream>>>(static_cast<const float*>(p.v), nullptr, static_cast<float*>(p.out),
                                       sink, L, p.hq, p.hkv, p.head_dim, epi);
  } else if (p.kv_dtype == FA_I8) {
    auto kern = empty_rows_kernel<int8_t, __nv_bfloat16>;
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<grid, 128, 0, ctx.stream>>>(static_cast<const int8_t*>(p.v), p.v_scales,
                                       static_cast<__nv_bfloat16*>(p.out), sink, L, p.hq, p.hkv, p.head_dim, epi);
  } else {
    auto kern = empty_rows_kernel<__nv_bfloat16, __nv_bfloat16>;
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<grid, 128, 0, ctx.stream>>>(static_cast<const __nv_bfloat16*>(p.v), nullptr,
                                       static_cast<__nv_bfloat16*>(p.out), sink, L, p.hq, p.hkv, p.head_dim, epi);
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace fa
