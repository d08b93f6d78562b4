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
#include <cuda_fp16.h>

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
  // two rows per iteration: their independent chains interleave
  for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row0 < rows;
       row0 += 2 * warps) {
    const int64_t rr[2] = {row0, row0 + warps};
    const bool live1 = rr[1] < rows;
    float v[2][E];
    load_row<E>(x + rr[0] * D + lane * E, v[0]);
    if (live1) {
      load_row<E>(x + rr[1] * D + lane * E, v[1]);
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) v[1][i] = 0.f;
    }
    float ss[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int i = 0; i < E; ++i) {
        v[r][i] *= sg[i];
        ss[r] = fmaf(v[r][i], v[r][i], ss[r]);
      }
#pragma unroll
    for (int h = 16; h > 0; h >>= 1) {
      ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], h);
      ss[1] += __shfl_xor_sync(0xffffffffu, ss[1], h);
    }
    warp_fwht<E>(v[0], lane);
    warp_fwht<E>(v[1], lane);
    uint32_t val[2];
    float norm[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      norm[r] = sqrtf(ss[r]);
      const float inv = norm[r] > 0.f ? inv_sqrt_d / norm[r] : 0.f;
      val[r] = 0;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float u = v[r][i] * inv;
        // the number of edges below u, by binary search (edges ascending)
        uint32_t c = 0;
#pragma unroll
        for (int h = NL / 2; h > 0; h >>= 1) c += (u > edge[c + h - 1]) ? h : 0u;
        val[r] |= c << (i * B);
      }
    }
    // word w of a row gathers the code bits of lanes l0 .. l0 + MAXC - 1
    const int w = lane;
    const int l0 = (32 * w) / LB;
    uint32_t word[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      const int src = min(l0 + j, 31);
      const uint32_t t0 = __shfl_sync(0xffffffffu, val[0], src);
      const uint32_t t1 = __shfl_sync(0xffffffffu, val[1], src);
      const int shift = src * LB - 32 * w;
      if (l0 + j <= 31 && shift < 32 && shift > -LB) {
        word[0] |= shift >= 0 ? (t0 << shift) : (t0 >> (-shift));
        word[1] |= shift >= 0 ? (t1 << shift) : (t1 >> (-shift));
      }
    }
    if (w < W) {
      reinterpret_cast<uint32_t*>(codes + rr[0] * (D * B / 8))[w] = word[0];
      if (live1) reinterpret_cast<uint32_t*>(codes + rr[1] * (D * B / 8))[w] = word[1];
    }
    if (lane == 0) {
      norms[rr[0]] = norm[0];
      if (live1) norms[rr[1]] = norm[1];
    }
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// Four 8x8 b16 matrices loaded transposed; lane l gives the row address of
// matrix l / 8, row l % 8.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// The 8x8 b16 matrix whose row g / 4, columns 2 (g % 4) .. +1 lane g holds,
// transposed (one movmatrix).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// D (fp32) += A (16x16 fp16, row) . B (16x8 fp16, col)
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four B-bit codes, one per nibble of `nib`, to fp16 pairs {level[c0],
// level[c1]} and {level[c2], level[c3]}.  The codebook is antisymmetric:
// with P the upper half of the levels (positive, ascending), a code c in the
// upper half reads P[c - half] and one in the lower half -P[half - 1 - c].
// pl / ph hold the low / high bytes of P[0..7] (fp16), so one byte permute
// per byte plane looks up four codes; the sign bit is ORed in after.
template <int B>
__device__ __forceinline__ void dequant4(uint32_t nib, const uint32_t (&pl)[2], const uint32_t (&ph)[2],
                                         uint32_t& h01, uint32_t& h23) {
  constexpr uint32_t kHalf = 1u << (B - 1);
  const uint32_t pos = (nib >> (B - 1)) & 0x1111u;
  const uint32_t neg = pos ^ 0x1111u;
  const uint32_t j = (nib & (0x1111u * (kHalf - 1))) ^ (neg * (kHalf - 1));
  const uint32_t lo = prmt(pl[0], pl[1], j);
  const uint32_t hi = prmt(ph[0], ph[1], j);
  h01 = prmt(lo, hi, 0x5140u) | ((neg & 0x1u) << 15) | ((neg & 0x10u) << 27);
  h23 = prmt(lo, hi, 0x7362u) | ((neg & 0x100u) << 7) | ((neg & 0x1000u) << 19);
}

// The 4B bits of four consecutive B-bit codes, one code per nibble.
template <int B>
__device__ __forceinline__ uint32_t to_nibbles(uint32_t f) {
  if constexpr (B == 4) {
    return f;
  } else if constexpr (B == 3) {
    return (f & 0x7u) | ((f & 0x38u) << 1) | ((f & 0x1c0u) << 2) | ((f & 0xe00u) << 3);
  } else {
    return (f & 0x3u) | ((f & 0xcu) << 2) | ((f & 0x30u) << 4) | ((f & 0xc0u) << 6);
  }
}

// Split-K decode over one (sequence, KV head, key split).  Per warp and
// 32-key chunk:
//   S^T [32 keys x 8 heads] = K_hat . (R q)^T on mma.sync m16n8k16 (keys on
//     M, the group's heads on N, channels on K).  Channels are summed over,
//     so their order inside a k-step is free: thread (g, t) takes channels
//     [t d/4, t d/4 + d/4) of its rows, four per k-step, and the rotated
//     queries' B fragments (fp16, registers) use the same order.  A
//     fragments come from the packed codes: with 4-bit codes each code byte
//     (two channels) indexes a table of fp16 level pairs in dynamic shared
//     memory, 32 KB with one copy per lane so every lane reads its own bank
//     (one load per fragment register); other widths by byte permutes
//     (dequant4).
//   online softmax per head on the S fragments; P'[key, head] = p ||v_key||
//     in fp16, turned from S fragments into B fragments by 8x8 transposes.
//   V: lane j dequantises key j's codes into an fp16 tile [32 keys x D] in
//     shared memory (a pair table of fp16 levels; 16-byte chunks of each row
//     swizzled by the key's low bits, so ldmatrix reads are conflict-free),
//     then O_rot^T [D x 8 heads] += Vlev^T . P' on mma.sync (channels on M,
//     heads on N, keys on K), the A fragments read by ldmatrix.trans.
// Three CTAs per SM: at most 168 registers a thread.
template <int D, int KB, int VB, int G>
__global__ void __launch_bounds__(kDecodeWarps * 32, 3)
    tq_decode_kernel(TqArgs A) {
  constexpr int E = D / 32;
  constexpr int KROW = D * KB / 8;  // bytes of a packed K row
  constexpr int VROW = D * VB / 8;
  constexpr int VU2 = VROW / 8;     // 8-byte words of a 32-key V block per lane
  constexpr int KS = D / 16;        // k-steps of the score MMA
  constexpr int SB = D * KB / 32;   // bytes of a thread's quarter of a K row
  constexpr int SW = (SB + 3) / 4;
  constexpr int MT = D / 16;        // channel tiles of the V MMA
  constexpr uint32_t kVdqBytes = kDecodeWarps * 32 * D * 2;      // fp16 V tiles of the warps
  constexpr uint32_t kSoBytes = kDecodeWarps * G * D * 4;         // the warps' O rows at the end
  __shared__ __align__(16) float qr[D][G];
  __shared__ uint32_t vtab[1 << (2 * VB)];  // V pair table: fp16 (level[c & m], level[c >> b])
  __shared__ __align__(16) uint2 vblk[kDecodeWarps][32 * VU2];  // a warp's staged V codes
  __shared__ float s_m[kDecodeWarps][G], s_l[kDecodeWarps][G];
  // the V tiles during the key loop, the per-warp O rows after it
  __shared__ __align__(128) unsigned char vbuf[kVdqBytes > kSoBytes ? kVdqBytes : kSoBytes];
  float(*s_o)[G][D] = reinterpret_cast<float(*)[G][D]>(vbuf);
  // 4-bit K codes: fp16 level pairs of every code byte, one copy per lane
  // (entry e of lane l at word 32 e + l), so each lane reads its own bank
  extern __shared__ __align__(16) uint32_t ktab[];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row group and column pair
  const int bg = blockIdx.y, split = blockIdx.x;
  const int b = bg / A.hkv, g = bg % A.hkv;
  int len = A.seqlens[b];
  if (len < 0 || len > A.cap) {
    if (threadIdx.x == 0 && split == 0 && g == 0) record_status(A.wd, kStatusRange);
    len = len < 0 ? 0 : A.cap;
  }
  const int k0 = split * A.split_keys;
  const int k1 = min(len, k0 + A.split_keys);
  for (int c = threadIdx.x; c < (1 << (2 * VB)); c += blockDim.x)
    vtab[c] = pack_h2(A.v_levels[c & ((1 << VB) - 1)], A.v_levels[c >> VB]);
  if constexpr (KB == 4) {
    if (k0 < k1) {
      for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const int e = i >> 5;
        ktab[i] = pack_h2(A.k_levels[e & 15], A.k_levels[e >> 4]);
      }
    }
  }
  // other widths: the upper half of the K levels as fp16 byte planes (8
  // entries, zero-padded)
  uint32_t pl[2] = {0u, 0u}, ph[2] = {0u, 0u};
#pragma unroll
  for (int jj = 0; jj < (1 << (KB - 1)); ++jj) {
    const __half hv = __float2half_rn(A.k_levels[(1 << (KB - 1)) + jj]);
    const uint32_t bits = *reinterpret_cast<const uint16_t*>(&hv);
    pl[jj / 4] |= (bits & 0xffu) << (8 * (jj % 4));
    ph[jj / 4] |= (bits >> 8) << (8 * (jj % 4));
  }
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
  // B fragments: head gq (zero past the group), channels t d/4 + 4 ks + 0..3
  uint32_t qb[KS][2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int ch = tq * (D / 4) + 4 * ks;
    const bool on = gq < G;
    const int hh = on ? gq : 0;
    qb[ks][0] = on ? pack_h2(qr[ch][hh], qr[ch + 1][hh]) : 0u;
    qb[ks][1] = on ? pack_h2(qr[ch + 2][hh], qr[ch + 3][hh]) : 0u;
  }

  float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};  // heads 2 tq, 2 tq + 1
  // O_rot^T fragments: channels 16 mi + gq (+ 8), heads 2 tq, 2 tq + 1
  float o[MT][4];
#pragma unroll
  for (int mi = 0; mi < MT; ++mi) o[mi][0] = o[mi][1] = o[mi][2] = o[mi][3] = 0.f;
  const uint32_t vdq = smem_u32(vbuf) + warp * (32 * D * 2);
  const int64_t plane = static_cast<int64_t>(b) * A.hkv + g;
  const uint8_t* kc = A.kc + plane * A.cap * KROW;
  const uint8_t* vc = A.vc + plane * A.cap * VROW;
  const float* kn = A.kn + plane * A.cap;
  const float* vn = A.vn + plane * A.cap;

  // one chunk's operands: the quarter K rows of this thread's four keys
  // (16 mt + gq + 8 r), their norms, and its share of the packed V rows
  auto load_chunk = [&](int c, uint32_t (&kw)[4][SW], float (&nk)[4], float (&nv)[4], uint2 (&vr)[VU2]) {
    const int n = k1 - c;
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
      const int kk = 16 * (r4 >> 1) + gq + 8 * (r4 & 1);
      nk[r4] = 0.f;
      nv[r4] = 0.f;
#pragma unroll
      for (int t = 0; t < SW; ++t) kw[r4][t] = 0u;
      if (kk < n) {
        const uint8_t* src = kc + static_cast<int64_t>(c + kk) * KROW + tq * SB;
        if constexpr (SB % 16 == 0) {
#pragma unroll
          for (int t = 0; t < SW / 4; ++t) {
            const uint4 u = reinterpret_cast<const uint4*>(src)[t];
            kw[r4][4 * t] = u.x; kw[r4][4 * t + 1] = u.y; kw[r4][4 * t + 2] = u.z; kw[r4][4 * t + 3] = u.w;
          }
        } else if constexpr (SB % 8 == 0) {
#pragma unroll
          for (int t = 0; t < SW / 2; ++t) {
            const uint2 u = reinterpret_cast<const uint2*>(src)[t];
            kw[r4][2 * t] = u.x; kw[r4][2 * t + 1] = u.y;
          }
        } else if constexpr (SB % 4 == 0) {
#pragma unroll
          for (int t = 0; t < SW; ++t) kw[r4][t] = reinterpret_cast<const uint32_t*>(src)[t];
        } else {  // 6-byte quarters (d = 64, 3 bits): 2-byte loads
          const uint16_t* h = reinterpret_cast<const uint16_t*>(src);
          kw[r4][0] = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
          kw[r4][1] = h[2];
        }
        nk[r4] = kn[c + kk];
        nv[r4] = vn[c + kk];
      }
    }
    const uint2* vsrc = reinterpret_cast<const uint2*>(vc + static_cast<int64_t>(c) * VROW);
#pragma unroll
    for (int t = 0; t < VU2; ++t) {
      const int idx = t * 32 + lane;
      vr[t] = (idx * 8) / VROW < n ? vsrc[idx] : make_uint2(0u, 0u);
    }
  };

  int c0 = k0 + warp * 32;
  uint32_t kw[4][SW];
  float nk[4], nv[4];
  uint2 vr[VU2];
  if (c0 < k1) load_chunk(c0, kw, nk, nv, vr);
  for (; c0 < k1; c0 += kDecodeWarps * 32) {
    __syncwarp();  // the previous chunk's reads of vblk and ps are done
#pragma unroll
    for (int t = 0; t < VU2; ++t) vblk[warp][t * 32 + lane] = vr[t];
    uint32_t kc4[4][SW];
    float nk4[4], nv4[4];
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
      nk4[r4] = nk[r4];
      nv4[r4] = nv[r4];
#pragma unroll
      for (int t = 0; t < SW; ++t) kc4[r4][t] = kw[r4][t];
    }
    // the next chunk's loads fly while this one computes
    const int c1 = c0 + kDecodeWarps * 32;
    if (c1 < k1) load_chunk(c1, kw, nk, nv, vr);

    // scores on the tensor cores: two 16-key tiles
    float sacc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int t = 0; t < 4; ++t) sacc[mt][t] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a0, a1, a2, a3;
        if constexpr (KB == 4) {
          // the code bytes of channels 4 ks .. +3: each byte is the table
          // index of its fp16 pair (offset 128 bytes per entry)
          const uint32_t* kt = ktab + lane;
          const uint32_t w0 = kc4[2 * mt][ks >> 1] >> (16 * (ks & 1));
          const uint32_t w1 = kc4[2 * mt + 1][ks >> 1] >> (16 * (ks & 1));
          a0 = kt[(w0 << 5) & 0x1fe0u];
          a2 = kt[(w0 >> 3) & 0x1fe0u];
          a1 = kt[(w1 << 5) & 0x1fe0u];
          a3 = kt[(w1 >> 3) & 0x1fe0u];
        } else {
          dequant4<KB>(to_nibbles<KB>(code_at<4 * KB, SW>(kc4[2 * mt], 4 * ks * KB)), pl, ph, a0, a2);
          dequant4<KB>(to_nibbles<KB>(code_at<4 * KB, SW>(kc4[2 * mt + 1], 4 * ks * KB)), pl, ph, a1, a3);
        }
        mma_f16(sacc[mt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
      }
    }
    // online softmax for heads 2 tq, 2 tq + 1 over the chunk's 32 keys
    float sv[2][4];
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int r4 = 2 * mt + (t >> 1);
        const int kk = 16 * mt + gq + 8 * (t >> 1);
        const float x = c0 + kk < k1 ? sacc[mt][t] * nk4[r4] : -INFINITY;
        sv[mt][t] = x;
        tmax[t & 1] = fmaxf(tmax[t & 1], x);
      }
    float alpha2[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float mx = tmax[hh];
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m2[hh], mx);
      alpha2[hh] = m2[hh] == -INFINITY ? 0.f : exp2f(m2[hh] - m_new);
      m2[hh] = m_new;
      l2[hh] *= alpha2[hh];
    }
    // P' = p ||v|| (0 for heads past the group) as B fragments of the V MMA:
    // the S fragment rows are keys and its columns heads; one transpose per
    // 8x8 gives thread (g, t) keys 2t, 2t + 1 of head g
    uint32_t pb[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float pv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int hh = t & 1;
        const int r4 = 2 * mt + (t >> 1);
        const float pe = sv[mt][t] == -INFINITY ? 0.f : exp2f(sv[mt][t] - m2[hh]);
        l2[hh] += pe;
        pv[t] = 2 * tq + hh < G ? pe * nv4[r4] : 0.f;
      }
      pb[mt][0] = transpose8x8(pack_h2(pv[0], pv[1]));
      pb[mt][1] = transpose8x8(pack_h2(pv[2], pv[3]));
    }
    // O columns (heads 2 tq, 2 tq + 1) take their alpha
#pragma unroll
    for (int mi = 0; mi < MT; ++mi) {
      o[mi][0] *= alpha2[0];
      o[mi][1] *= alpha2[1];
      o[mi][2] *= alpha2[0];
      o[mi][3] *= alpha2[1];
    }
    __syncwarp();
    // V: lane j dequantises key j (codes of keys past the chunk's end are
    // zero, and their P' is 0), then the MMAs over the two 16-key halves
    {
      constexpr int NW = VROW / 4;
      uint32_t vw[NW];
      const uint32_t* row = reinterpret_cast<const uint32_t*>(vblk[warp]) + lane * NW;
#pragma unroll
      for (int t = 0; t < NW; ++t) vw[t] = row[t];
#pragma unroll
      for (int c16 = 0; c16 < D / 8; ++c16) {  // 8 channels = four level pairs per 16-byte chunk
        uint32_t h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) h[q] = vtab[code_at<2 * VB, NW>(vw, (8 * c16 + 2 * q) * VB)];
        const uint32_t at = vdq + lane * (D * 2) + ((c16 ^ (lane & 7)) * 16);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(at), "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                     : "memory");
      }
      __syncwarp();
      // ldmatrix.trans of 8x8 block i = lane / 8: keys 8 (i / 2) + lane % 8 of
      // the 16-key half, channels 16 mi + 8 (i % 2) ..
      const int blk = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int key = 16 * mt + 8 * (blk >> 1) + rr;
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
          const int c16 = 2 * mi + (blk & 1);
          uint32_t a[4];
          ldsm_x4_trans(vdq + key * (D * 2) + ((c16 ^ (key & 7)) * 16), a);
          mma_f16(o[mi], a[0], a[1], a[2], a[3], pb[mt][0], pb[mt][1]);
        }
      }
    }
  }

  // this warp's state: m and l of head 2 tq + hh sit in the lanes of column
  // pair tq (l summed over them); O in the lanes over the channels
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float l = l2[hh];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    const int h = 2 * tq + hh;
    if (gq == 0 && h < G) {
      s_m[warp][h] = m2[hh];
      s_l[warp][h] = l;
    }
  }
  __syncthreads();  // every warp's V tile reads are done: vbuf becomes the O rows
#pragma unroll
  for (int mi = 0; mi < MT; ++mi) {
    const int c = 16 * mi + gq;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = 2 * tq + hh;
      if (h < G) {
        s_o[warp][h][c] = o[mi][hh];
        s_o[warp][h][c + 8] = o[mi][2 + hh];
      }
    }
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
  // 4-bit K: the replicated pair table in dynamic shared memory
  constexpr int kDyn = KB == 4 ? 256 * 32 * 4 : 0;
  auto go = [&](auto kern) {
    note_variant(reinterpret_cast<const void*>(kern));
    if (kDyn > 0 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDyn) != cudaSuccess)
      return FA_ERR_CUDA;
    kern<<<grid, kDecodeWarps * 32, kDyn, st>>>(A);
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
    const int64_t need = (p.rows + 15) / 16;  // eight warps, two rows per warp per pass
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
