// turboquant.cu -- TurboQuant KV cache compression and decode over it.
//
// What it computes (the C attention library's README, "TurboQuant KV Cache
// Compression"): each K or V row of head size d is rotated by a randomized
// Hadamard transform, random +-1 signs applied before the transform,
//   y = H (s * x) / sqrt(d)      (H Sylvester-ordered, orthonormal after the scale),
// normalised by its L2 norm, u = y / ||x||, each coordinate of u quantised to
// b = 2..4 bits by the Lloyd-Max quantiser of the Beta(d/2, d/2) law of
// (u + 1) / 2, and the codes bit-packed (channel i at bits [i b, i b + b) of
// the row's little-endian bit stream) beside one fp32 norm per row.
//
// Decode never rebuilds K or V.  With R the rotation, q . k_hat = ||k|| (R q)
// . level[code], so q is rotated once per head and each key costs a table
// lookup and an FMA per channel; the V side accumulates sum_j p_j ||v_j||
// level[code_j] in the rotated basis and the merge kernel applies R^T once per
// output row.
//
// Kernels: tq_compress_kernel (one warp per row: loads, signs, the in-lane
// and cross-lane butterflies of the transform, the norm, the code decisions
// and the packing of 32-bit words by shuffles), tq_decode_kernel (split-K:
// one CTA of four warps per (sequence, KV head, key split); scores with one
// key per lane, the V update with the lanes over the channels), and
// tq_merge_kernel (one warp per output row: the split merge, the inverse
// rotation, the epilogue, the bf16 store).
#include <cmath>
#include <vector>

#include "internal.h"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kDecodeWarps = 4;

// ---------------------------------------------------------------- helpers
template <int E>
__device__ __forceinline__ void load_row(const float* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  }
}
template <int E>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const uint2 t = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
  } else {
    const uint32_t t = *reinterpret_cast<const uint32_t*>(p);
    v[0] = __uint_as_float(t << 16); v[1] = __uint_as_float(t & 0xffff0000u);
  }
}

// Unnormalised Walsh-Hadamard transform of a warp-held vector: lane l holds
// elements [l E, l E + E).  Strides below E stay in the lane; stride h E
// pairs lane l with lane l ^ h.  The lower element of a pair takes a + b,
// the upper one a - b (a the lower, b the upper).
template <int E>
__device__ __forceinline__ void warp_fwht(float (&v)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], h);
      v[i] = (lane & h) ? other - v[i] : v[i] + other;
    }
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int h = 16; h > 0; h >>= 1) x += __shfl_xor_sync(0xffffffffu, x, h);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int h = 16; h > 0; h >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, h));
  return x;
}

// b-bit code starting at bit `pos` of the little-endian word array w (pos
// and B compile-time after unrolling; a code may straddle two words).
template <int B, int NW>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[NW], int pos) {
  const int k = pos >> 5, sh = pos & 31;
  uint32_t x = w[k] >> sh;
  if (sh + B > 32) x = __funnelshift_r(w[k], w[k + 1], sh);
  return x & ((1u << B) - 1u);
}

// ---------------------------------------------------------------- compress
template <int D, int B, typename T>
__global__ void __launch_bounds__(256)
    tq_compress_kernel(const T* __restrict__ x, int64_t rows, const float* __restrict__ signs,
                       const float* __restrict__ levels, uint8_t* __restrict__ codes, float* __restrict__ norms) {
  constexpr int E = D / 32;            // channels per lane
  constexpr int NL = 1 << B;           // levels
  constexpr int W = D * B / 32;        // 32-bit words per packed row
  constexpr int LB = E * B;            // code bits per lane
  constexpr int MAXC = (32 + LB - 1) / LB + 1;  // lanes feeding one word
  const int lane = threadIdx.x & 31;
  // cell edges, with a sentinel so the binary search below reads edge[c + h - 1]
  __shared__ float edge[NL];
  if (threadIdx.x < NL - 1) edge[threadIdx.x] = 0.5f * (levels[threadIdx.x] + levels[threadIdx.x + 1]);
  if (threadIdx.x == NL - 1) edge[NL - 1] = INFINITY;
  __syncthreads();
  float sg[E];
#pragma unroll
  for (int i = 0; i < E; ++i) sg[i] = signs[lane * E + i];
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    float v[E];
    load_row<E>(x + row * D + lane * E, v);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      v[i] *= sg[i];
      ss = fmaf(v[i], v[i], ss);
    }
    ss = warp_sum(ss);
    warp_fwht<E>(v, lane);
    const float norm = sqrtf(ss);
    const float inv = norm > 0.f ? inv_sqrt_d / norm : 0.f;
    uint32_t val = 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float u = v[i] * inv;
      // the number of edges below u, by binary search (edges ascending)
      uint32_t c = 0;
#pragma unroll
      for (int h = NL / 2; h > 0; h >>= 1) c += (u > edge[c + h - 1]) ? h : 0u;
      val |= c << (i * B);
    }
    // word w of the row gathers the code bits of lanes l0 .. l0 + MAXC - 1
    const int w = lane;
    const int l0 = (32 * w) / LB;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      const int src = min(l0 + j, 31);
      const uint32_t t = __shfl_sync(0xffffffffu, val, src);
      const int shift = src * LB - 32 * w;
      if (l0 + j <= 31 && shift < 32 && shift > -LB)
        word |= shift >= 0 ? (t << shift) : (t >> (-shift));
    }
    if (w < W) reinterpret_cast<uint32_t*>(codes + row * (D * B / 8))[w] = word;
    if (lane == 0) norms[row] = norm;
  }
}

// ---------------------------------------------------------------- decode
struct TqArgs {
  const __nv_bfloat16* q;
  const uint8_t* kc;
  const float* kn;
  const uint8_t* vc;
  const float* vn;
  const float* k_levels;
  const float* v_levels;
  const float* signs;
  const int* seqlens;
  float* part;  // [batch*hq, nsplit, D + 2]: unnormalised rotated o, m (log2 units), l
  int hq, hkv, cap, split_keys, nsplit;
  float scale_log2;
  Watchdog wd;
};

template <int D, int KB, int VB, int G>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    tq_decode_kernel(TqArgs A) {
  constexpr int E = D / 32;
  constexpr int KW = D * KB / 32;   // 32-bit words of a packed K row
  constexpr int KROW = D * KB / 8;  // bytes of a packed K row
  constexpr int VROW = D * VB / 8;
  constexpr int LVB = E * VB;       // V code bits per lane (its E channels)
  constexpr int VU2 = VROW / 8;     // 8-byte words of a 32-key V block per lane
  constexpr int GP = (G + 1) / 2;   // head pairs
  // queries interleaved by head: one vector load gives a channel of every head
  __shared__ __align__(16) float qr[D][G];
  // V pair table: entry c is (level[c & m], level[c >> b]) for two consecutive
  // b-bit codes read as one 2b-bit field
  __shared__ float klut[1 << KB];  // one code per read: distinct entries, distinct banks
  __shared__ __align__(8) float2 vtab[1 << (2 * VB)];
  __shared__ __align__(16) uint2 vblk[kDecodeWarps][32 * VU2];  // a warp's staged V codes
  __shared__ float s_m[kDecodeWarps][G], s_l[kDecodeWarps][G];
  __shared__ __align__(16) float s_o[kDecodeWarps][G][D];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bg = blockIdx.y, split = blockIdx.x;
  const int b = bg / A.hkv, g = bg % A.hkv;
  int len = A.seqlens[b];
  if (len < 0 || len > A.cap) {
    if (threadIdx.x == 0 && split == 0 && g == 0) record_status(A.wd, kStatusRange);
    len = len < 0 ? 0 : A.cap;
  }
  const int k0 = split * A.split_keys;
  const int k1 = min(len, k0 + A.split_keys);
  if (threadIdx.x < (1 << KB)) klut[threadIdx.x] = A.k_levels[threadIdx.x];
  for (int c = threadIdx.x; c < (1 << (2 * VB)); c += blockDim.x)
    vtab[c] = make_float2(A.v_levels[c & ((1 << VB) - 1)], A.v_levels[c >> VB]);
  // rotated, pre-scaled queries: qr = scale log2(e) H (s * q) / sqrt(d)
  for (int gi = warp; gi < G; gi += kDecodeWarps) {
    const int h = g * G + gi;
    float v[E];
    load_row<E>(A.q + (static_cast<int64_t>(b) * A.hq + h) * D + lane * E, v);
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] *= A.signs[lane * E + i];
    warp_fwht<E>(v, lane);
    const float sc = A.scale_log2 * rsqrtf(static_cast<float>(D));
#pragma unroll
    for (int i = 0; i < E; ++i) qr[lane * E + i][gi] = v[i] * sc;
  }
  __syncthreads();

  float m[G], lsum[G];
  float2 o[GP][E];  // heads (2p, 2p + 1) of channel e of this lane
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    m[gi] = -INFINITY;
    lsum[gi] = 0.f;
  }
#pragma unroll
  for (int pi = 0; pi < GP; ++pi)
#pragma unroll
    for (int e = 0; e < E; ++e) o[pi][e] = make_float2(0.f, 0.f);
  const int64_t plane = static_cast<int64_t>(b) * A.hkv + g;
  const uint8_t* kc = A.kc + plane * A.cap * KROW;
  const uint8_t* vc = A.vc + plane * A.cap * VROW;
  const float* kn = A.kn + plane * A.cap;
  const float* vn = A.vn + plane * A.cap;

  // one chunk's operands: this lane's K row and both norms of its key, and
  // its share of the chunk's packed V rows (rows past the end read as 0)
  auto load_chunk = [&](int c, uint32_t (&kw)[KW], float& nk, float& nv, uint2 (&vr)[VU2]) {
    const int key = c + lane;
    const int n = k1 - c;
    nk = 0.f;
    nv = 0.f;
    if (key < k1) {
      if constexpr (KROW % 16 == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(kc + static_cast<int64_t>(key) * KROW);
#pragma unroll
        for (int t = 0; t < KW / 4; ++t) {
          const uint4 u = src[t];
          kw[4 * t] = u.x; kw[4 * t + 1] = u.y; kw[4 * t + 2] = u.z; kw[4 * t + 3] = u.w;
        }
      } else {  // 24-byte rows (d = 64, 3 bits): 8-byte loads
        const uint2* src = reinterpret_cast<const uint2*>(kc + static_cast<int64_t>(key) * KROW);
#pragma unroll
        for (int t = 0; t < KW / 2; ++t) {
          const uint2 u = src[t];
          kw[2 * t] = u.x; kw[2 * t + 1] = u.y;
        }
      }
      nk = kn[key];
      nv = vn[key];
    } else {
#pragma unroll
      for (int t = 0; t < KW; ++t) kw[t] = 0u;
    }
    const uint2* vsrc = reinterpret_cast<const uint2*>(vc + static_cast<int64_t>(c) * VROW);
#pragma unroll
    for (int t = 0; t < VU2; ++t) {
      const int idx = t * 32 + lane;
      vr[t] = (idx * 8) / VROW < n ? vsrc[idx] : make_uint2(0u, 0u);
    }
  };

  int c0 = k0 + warp * 32;
  uint32_t kw[KW];
  float nk = 0.f, nv = 0.f;
  uint2 vr[VU2];
  if (c0 < k1) load_chunk(c0, kw, nk, nv, vr);
  for (; c0 < k1; c0 += kDecodeWarps * 32) {
    __syncwarp();
#pragma unroll
    for (int t = 0; t < VU2; ++t) vblk[warp][t * 32 + lane] = vr[t];
    const float nk_c = nk, nv_c = nv;
    uint32_t kw_c[KW];
#pragma unroll
    for (int t = 0; t < KW; ++t) kw_c[t] = kw[t];
    // the next chunk's loads fly while this one computes
    const int c1 = c0 + kDecodeWarps * 32;
    if (c1 < k1) load_chunk(c1, kw, nk, nv, vr);

    // scores: one key per lane, two channels per table read
    const int key = c0 + lane;
    float acc[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) acc[gi] = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      const float lv = klut[code_at<KB, KW>(kw_c, i * KB)];
      if constexpr (G == 1) {
        acc[0] = fmaf(qr[i][0], lv, acc[0]);
      } else if constexpr (G == 2) {
        const float2 q2 = *reinterpret_cast<const float2*>(&qr[i][0]);
        const float2 a = fma2(q2, make_float2(lv, lv), make_float2(acc[0], acc[1]));
        acc[0] = a.x;
        acc[1] = a.y;
      } else {
        // four heads per 16-byte broadcast read of the rotated queries
#pragma unroll
        for (int g4 = 0; g4 < G; g4 += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(&qr[i][g4]);
          const float2 a = fma2(make_float2(q4.x, q4.y), make_float2(lv, lv), make_float2(acc[g4], acc[g4 + 1]));
          const float2 c = fma2(make_float2(q4.z, q4.w), make_float2(lv, lv), make_float2(acc[g4 + 2], acc[g4 + 3]));
          acc[g4] = a.x;
          acc[g4 + 1] = a.y;
          acc[g4 + 2] = c.x;
          acc[g4 + 3] = c.y;
        }
      }
    }
    // online softmax, per head, over this warp's 32 keys; p carries ||v||
    float p[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      const float s = key < k1 ? acc[gi] * nk_c : -INFINITY;
      const float m_new = fmaxf(m[gi], warp_max(s));
      const float alpha = m[gi] == -INFINITY ? 0.f : exp2f(m[gi] - m_new);
      const float pe = s == -INFINITY ? 0.f : exp2f(s - m_new);
      lsum[gi] = lsum[gi] * alpha + pe;
      m[gi] = m_new;
      p[gi] = pe * nv_c;
      if (alpha != 1.f) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if (gi % 2 == 0) o[gi / 2][e].x *= alpha;
          else o[gi / 2][e].y *= alpha;
        }
      }
    }
    __syncwarp();
    // V: the lanes over the channels, one key at a time
    const int n = min(32, k1 - c0);
    const int bitpos = lane * LVB;
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(vblk[warp]) + (bitpos >> 5);
    const int sh = bitpos & 31;
    const bool two = sh + LVB > 32;  // this lane's bits cross into the next word
    for (int j = 0; j < n; ++j) {
      const uint32_t w0 = vw[j * (VROW / 4)];
      const uint32_t w1 = two ? vw[j * (VROW / 4) + 1] : 0u;
      const uint32_t bits = __funnelshift_r(w0, w1, sh);
      float lev[E];
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        const float2 t = vtab[(bits >> (e * VB)) & ((1u << (2 * VB)) - 1u)];
        lev[e] = t.x;
        lev[e + 1] = t.y;
      }
#pragma unroll
      for (int pi = 0; pi < GP; ++pi) {
        const float p0 = __shfl_sync(0xffffffffu, p[2 * pi], j);
        const float p1 = (2 * pi + 1 < G) ? __shfl_sync(0xffffffffu, p[(2 * pi + 1) % G], j) : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) o[pi][e] = fma2(make_float2(p0, p1), make_float2(lev[e], lev[e]), o[pi][e]);
      }
    }
  }

  // the four warps' states merge into this split's partial
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    const float l = warp_sum(lsum[gi]);
    if (lane == 0) {
      s_m[warp][gi] = m[gi];
      s_l[warp][gi] = l;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[warp][gi][lane * E + e] = gi % 2 == 0 ? o[gi / 2][e].x : o[gi / 2][e].y;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * (D + 2); idx += blockDim.x) {
    const int gi = idx / (D + 2), c = idx % (D + 2);
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) mx = fmaxf(mx, s_m[w][gi]);
    float r = 0.f;
    if (c == D) {
      r = mx;
    } else {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        if (s_m[w][gi] == -INFINITY) continue;
        const float f = exp2f(s_m[w][gi] - mx);
        r = fmaf(c < D ? s_o[w][gi][c] : s_l[w][gi], f, r);
      }
    }
    const int64_t row = static_cast<int64_t>(b) * A.hq + g * G + gi;
    A.part[(row * A.nsplit + split) * (D + 2) + c] = r;
  }
}

template <int D>
__global__ void __launch_bounds__(256)
    tq_merge_kernel(const float* __restrict__ part, int64_t rows, int nsplit, const float* __restrict__ signs,
                    __nv_bfloat16* __restrict__ out, Epilogue epi) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* pr = part + row * nsplit * (D + 2);
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, pr[s * (D + 2) + D]);
  float acc[E], l = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float ms = pr[s * (D + 2) + D];
      if (ms == -INFINITY) continue;
      const float f = exp2f(ms - mx);
      l = fmaf(pr[s * (D + 2) + D + 1], f, l);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(pr[s * (D + 2) + lane * E + e], f, acc[e]);
    }
  }
  // a sequence without cached keys gets o = 0
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] *= inv_l;
  warp_fwht<E>(acc, lane);  // back from the rotated basis: s * (H o) / sqrt(d)
  const float sc = rsqrtf(static_cast<float>(D));
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float y = apply_epilogue(acc[e] * sc * signs[lane * E + e], epi);
    out[row * D + lane * E + e] = __float2bfloat16_rn(y);
  }
}

template <int D, int KB, int VB>
fa_status launch_decode_g(const TqArgs& A, int group, dim3 grid, cudaStream_t st) {
  auto go = [&](auto kern) {
    note_variant(reinterpret_cast<const void*>(kern));
    kern<<<grid, kDecodeWarps * 32, 0, st>>>(A);
    return cuda_status(cudaGetLastError());
  };
  switch (group) {
    case 1: return go(tq_decode_kernel<D, KB, VB, 1>);
    case 2: return go(tq_decode_kernel<D, KB, VB, 2>);
    case 4: return go(tq_decode_kernel<D, KB, VB, 4>);
    case 8: return go(tq_decode_kernel<D, KB, VB, 8>);
  }
  return FA_ERR_UNSUPPORTED;
}

template <int D, int KB>
fa_status launch_decode_v(const TqArgs& A, int vb, int group, dim3 grid, cudaStream_t st) {
  switch (vb) {
    case 2: return launch_decode_g<D, KB, 2>(A, group, grid, st);
    case 3: return launch_decode_g<D, KB, 3>(A, group, grid, st);
    case 4: return launch_decode_g<D, KB, 4>(A, group, grid, st);
  }
  return FA_ERR_UNSUPPORTED;
}

template <int D>
fa_status launch_decode_d(const TqArgs& A, int kb, int vb, int group, dim3 grid, cudaStream_t st) {
  switch (kb) {
    case 2: return launch_decode_v<D, 2>(A, vb, group, grid, st);
    case 3: return launch_decode_v<D, 3>(A, vb, group, grid, st);
    case 4: return launch_decode_v<D, 4>(A, vb, group, grid, st);
  }
  return FA_ERR_UNSUPPORTED;
}

template <int D, typename T>
fa_status launch_compress_d(const fa_tq_compress_params& p, const LaunchCtx& ctx) {
  auto go = [&](auto kern) {
    note_variant(reinterpret_cast<const void*>(kern));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess || per_sm < 1)
      return FA_ERR_CUDA;
    const int64_t need = (p.rows + 7) / 8;
    const int64_t cap = static_cast<int64_t>(per_sm) * device_sm_count();
    const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
    kern<<<grid, 256, 0, ctx.stream>>>(static_cast<const T*>(p.x), p.rows, p.signs, p.levels, p.codes, p.norms);
    return cuda_status(cudaGetLastError());
  };
  switch (p.bits) {
    case 2: return go(tq_compress_kernel<D, 2, T>);
    case 3: return go(tq_compress_kernel<D, 3, T>);
    case 4: return go(tq_compress_kernel<D, 4, T>);
  }
  return FA_ERR_UNSUPPORTED;
}

}  // namespace

int tq_decode_splits(int capacity) { return (capacity + kTqSplitKeys - 1) / kTqSplitKeys; }

fa_status launch_tq_compress(const fa_tq_compress_params& p, const LaunchCtx& ctx) {
  if (p.rows == 0) return FA_OK;
  const bool bf = p.x_dtype == FA_BF16;
  if (p.head_dim == 128) return bf ? launch_compress_d<128, __nv_bfloat16>(p, ctx) : launch_compress_d<128, float>(p, ctx);
  if (p.head_dim == 64) return bf ? launch_compress_d<64, __nv_bfloat16>(p, ctx) : launch_compress_d<64, float>(p, ctx);
  return FA_ERR_UNSUPPORTED;
}

fa_status launch_tq_decode(const fa_tq_decode_params& p, float* part, const LaunchCtx& ctx) {
  if (p.batch == 0) return FA_OK;
  TqArgs A;
  A.q = static_cast<const __nv_bfloat16*>(p.q);
  A.kc = p.k_codes;
  A.kn = p.k_norms;
  A.vc = p.v_codes;
  A.vn = p.v_norms;
  A.k_levels = p.k_levels;
  A.v_levels = p.v_levels;
  A.signs = p.signs;
  A.seqlens = p.cache_seqlens;
  A.part = part;
  A.hq = p.hq;
  A.hkv = p.hkv;
  A.cap = p.capacity;
  A.split_keys = kTqSplitKeys;
  A.nsplit = tq_decode_splits(p.capacity);
  A.scale_log2 = p.softmax_scale * kLog2e;
  A.wd = ctx.wd;
  const dim3 grid(static_cast<unsigned>(A.nsplit), static_cast<unsigned>(p.batch * p.hkv));
  const int group = p.hq / p.hkv;
  fa_status st = p.head_dim == 128 ? launch_decode_d<128>(A, p.k_bits, p.v_bits, group, grid, ctx.stream)
                                   : launch_decode_d<64>(A, p.k_bits, p.v_bits, group, grid, ctx.stream);
  if (st != FA_OK) return st;
  const int64_t rows = static_cast<int64_t>(p.batch) * p.hq;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  const Epilogue epi = make_epilogue(p.epilogue, p.n_epilogue);
  auto merge = p.head_dim == 128 ? tq_merge_kernel<128> : tq_merge_kernel<64>;
  note_variant(reinterpret_cast<const void*>(merge));
  merge<<<blocks, 256, 0, ctx.stream>>>(part, rows, A.nsplit, p.signs, static_cast<__nv_bfloat16*>(p.out), epi);
  return cuda_status(cudaGetLastError());
}

// Lloyd-Max levels of u on [-1, 1] with density proportional to
// (1 - u^2)^(d/2 - 1) (u = 2t - 1, t ~ Beta(d/2, d/2)): the cumulative
// integrals of f and u f by the trapezoid rule on 2^20 intervals, read at the
// cell edges by linear interpolation; Lloyd's iteration (levels the cell
// centroids, edges the midpoints) from the quantiles at the cell centres;
// the result made exactly antisymmetric.
fa_status tq_codebook_host(int d, int bits, float* levels) {
  const int n = 1 << bits;
  const int N = 1 << 20;
  const double h = 2.0 / N, e = d / 2.0 - 1.0;
  std::vector<double> F0(N + 1), F1(N + 1);
  F0[0] = F1[0] = 0.0;
  double f_prev = 0.0, u_prev = -1.0;
  for (int k = 1; k <= N; ++k) {
    const double u = -1.0 + k * h;
    const double f = (k == N) ? 0.0 : std::pow(1.0 - u * u, e);
    F0[k] = F0[k - 1] + 0.5 * h * (f_prev + f);
    F1[k] = F1[k - 1] + 0.5 * h * (u_prev * f_prev + u * f);
    f_prev = f;
    u_prev = u;
  }
  auto at = [&](const std::vector<double>& F, double u) {
    double pos = (u + 1.0) / h;
    if (pos <= 0.0) return F[0];
    if (pos >= N) return F[N];
    const int k = static_cast<int>(pos);
    const double fr = pos - k;
    return F[k] + fr * (F[k + 1] - F[k]);
  };
  std::vector<double> lv(n), edge(n + 1);
  // quantiles at (i + 1/2) / n by bisection on the cumulative mass
  for (int i = 0; i < n; ++i) {
    const double target = (i + 0.5) / n * F0[N];
    double lo = -1.0, hi = 1.0;
    for (int it = 0; it < 200; ++it) {
      const double mid = 0.5 * (lo + hi);
      (at(F0, mid) < target ? lo : hi) = mid;
    }
    lv[i] = 0.5 * (lo + hi);
  }
  for (int it = 0; it < 200000; ++it) {
    edge[0] = -1.0;
    edge[n] = 1.0;
    for (int i = 1; i < n; ++i) edge[i] = 0.5 * (lv[i - 1] + lv[i]);
    double change = 0.0;
    for (int i = 0; i < n; ++i) {
      const double m0 = at(F0, edge[i + 1]) - at(F0, edge[i]);
      const double m1 = at(F1, edge[i + 1]) - at(F1, edge[i]);
      if (!(m0 > 0.0)) return FA_ERR_UNSUPPORTED;
      const double c = m1 / m0;
      change = std::fmax(change, std::fabs(c - lv[i]));
      lv[i] = c;
    }
    if (change < 1e-14) break;
  }
  for (int i = 0; i < n / 2; ++i) {
    const double a = 0.5 * (lv[n - 1 - i] - lv[i]);
    levels[i] = static_cast<float>(-a);
    levels[n - 1 - i] = static_cast<float>(a);
  }
  return FA_OK;
}

}  // namespace fa
