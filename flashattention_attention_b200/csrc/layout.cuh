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
  const int32_t* cu_q;  // null for dense queries
  const int32_t* cu_k;  // null for dense keys; per-sequence key counts otherwise
  int32_t s_q, s_k;     // dense lengths
  int32_t causal, window;
  // paged K/V (null table: rows as above): pools [num_pages, hkv, page_size, d];
  // key j of sequence b is row j % page_size of page block_table[b][j / page_size]
  const int32_t* block_table;
  int32_t max_pages, page_size, num_pages, hkv;

  static SeqLayout from(const fa_fwd_params& p) {
    SeqLayout L;
    L.block_table = nullptr;
    L.max_pages = L.page_size = L.num_pages = 0;
    L.hkv = p.hkv;
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
  // Queries as in `from`; keys in page pools, sequence b holding
  // cu_seqlens_k[b+1] - cu_seqlens_k[b] of them.
  static SeqLayout paged(const fa_fwd_params& p, const fa_kv_pages& pg) {
    SeqLayout L = from(p);
    L.cu_k = p.cu_seqlens_k;
    L.k_bstride = L.k_hstride = 0;
    L.block_table = pg.block_table;
    L.max_pages = pg.max_pages;
    L.page_size = pg.page_size;
    L.num_pages = pg.num_pages;
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
    s.s_q = L.cu_q[b + 1] - static_cast<int32_t>(q0);
  } else {
    s.s_q = L.s_q;
  }
  if (L.cu_k != nullptr) {
    k0 = L.cu_k[b];
    s.s_k = L.cu_k[b + 1] - static_cast<int32_t>(k0);
  } else {
    s.s_k = L.s_k;
  }
  s.q_row0 = L.q_bstride * b + L.q_hstride * h + q0;
  s.k_row0 = L.k_bstride * b + L.k_hstride * g + k0;
  return s;
}

// Paged keys: plane (page * hkv + g) and row inside it of key j of sequence
// b.  A page id outside the pool reads as page 0 (never outside the pool);
// `bad` reports it.
__device__ __forceinline__ void paged_key(const SeqLayout& L, int b, int g, int j, int& plane, int& row,
                                          bool& bad) {
  int pg = L.block_table[static_cast<int64_t>(b) * L.max_pages + j / L.page_size];
  bad = pg < 0 || pg >= L.num_pages;
  if (bad) pg = 0;
  plane = pg * L.hkv + g;
  row = j % L.page_size;
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
