// layout.cuh -- row addressing of the dense and varlen layouts and the
// visible-key band of a query row.
//
// Dense:  q/out row (b, h, i) = (b*hq + h)*s_q + i;  k/v row (b, g, j) = (b*hkv + g)*s_k + j
// Varlen: q/out row (b, h, i) = h*total_q + cu_q[b] + i;  k/v row = g*total_k + cu_k[b] + j
// Both are  row = bstride*b + hstride*h + start[b] + i.
//
// Band (fkl_python PR #6, Summary: causal flag; SKaiNET-transformers PR #419,
// Summary: sliding-window layers; bottom-right alignment): query i of a
// sequence with s_q queries and s_k keys sits at p = i + s_k - s_q and sees
// keys j with  0 <= j < s_k,  j <= p (causal),  j > p - window (window > 0).
#pragma once

#include <stdint.h>

#include "fa.h"

namespace fa {

struct SeqLayout {
  int64_t q_bstride, q_hstride, k_bstride, k_hstride;
  const int32_t* cu_q;  // null for dense
  const int32_t* cu_k;
  int32_t s_q, s_k;     // dense lengths
  int32_t causal, window;

  static SeqLayout from(const fa_fwd_params& p) {
    SeqLayout L;
    if (p.cu_seqlens_q == nullptr) {
      L.q_bstride = static_cast<int64_t>(p.hq) * p.seqlen_q;
      L.q_hstride = p.seqlen_q;
      L.k_bstride = static_cast<int64_t>(p.hkv) * p.seqlen_k;
      L.k_hstride = p.seqlen_k;
      L.cu_q = L.cu_k = nullptr;
    } else {
      L.q_bstride = 0;
      L.q_hstride = p.total_q;
      L.k_bstride = 0;
      L.k_hstride = p.total_k;
      L.cu_q = p.cu_seqlens_q;
      L.cu_k = p.cu_seqlens_k != nullptr ? p.cu_seqlens_k : p.cu_seqlens_q;
    }
    L.s_q = p.seqlen_q;
    L.s_k = p.seqlen_k;
    L.causal = p.causal;
    L.window = p.window;
    return L;
  }
};

struct Seq {
  int64_t q_row0;  // row of (b, h, 0)
  int64_t k_row0;  // row of (b, g, 0)
  int32_t s_q, s_k;
};

__device__ __forceinline__ Seq seq_of(const SeqLayout& L, int b, int h, int g) {
  Seq s;
  int64_t q0 = 0, k0 = 0;
  if (L.cu_q != nullptr) {
    q0 = L.cu_q[b];
    k0 = L.cu_k[b];
    s.s_q = L.cu_q[b + 1] - static_cast<int32_t>(q0);
    s.s_k = L.cu_k[b + 1] - static_cast<int32_t>(k0);
  } else {
    s.s_q = L.s_q;
    s.s_k = L.s_k;
  }
  s.q_row0 = L.q_bstride * b + L.q_hstride * h + q0;
  s.k_row0 = L.k_bstride * b + L.k_hstride * g + k0;
  return s;
}

// Visible key range [lo, hi) of query row i (lo >= hi: empty band).
__device__ __forceinline__ void band_of(const SeqLayout& L, int i, int s_q, int s_k, int& lo, int& hi) {
  const int p = i + s_k - s_q;
  hi = L.causal ? min(s_k, p + 1) : s_k;
  lo = L.window > 0 ? max(0, p - L.window + 1) : 0;
}

__device__ __forceinline__ bool visible(const SeqLayout& L, int i, int j, int s_q, int s_k) {
  const int p = i + s_k - s_q;
  if (j < 0 || j >= s_k) return false;
  if (L.causal && j > p) return false;
  if (L.window > 0 && j <= p - L.window) return false;
  return true;
}

}  // namespace fa
