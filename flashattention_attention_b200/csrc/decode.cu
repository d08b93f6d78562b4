// decode.cu -- single-query decode over a KV cache, split along the keys
// (fkl_python PR #6, Verification: "FA decode step s_q=1 vs s_k=256 int8";
// Summary: the int8 cache is dequantised in-register and never inflated in
// global memory; kernbench2 commit ADR-0060: decode splits the keys and
// reduces the partial softmax states (m, l, O) to one output).
//
// Work unit: (split, kv-head g, sequence b).  One CTA of 4 warps owns a
// split; each warp streams 32-key tiles of K codes, V codes and their fp32
// scales through its own 3-stage ring (TMA, 128-byte swizzle, bounded
// mbarrier waits), so a warp never waits on another warp.  All G = hq/hkv
// query heads of the group are served by every key read.
//
// Per tile (tensor cores through mma.sync m16n8k16, fp16 in, fp32 accumulate):
//   S^T[32 keys x 8 heads] = K_codes[32 x d] . Q^T    (keys on M, heads on N)
//   x = S * s_k[key] * scale * log2(e) * 2^-e_h        (K scale on S columns)
//   online softmax per head (running m, l in fp32, exp2)
//   P'[key, h] = p * s_v[key]                          (V scale on P rows; l sums p)
//   O^T[d x 8 heads] += V_codes^T[d x 32] . P'
// int8 codes convert exactly to fp16 with one LOP3 and one packed subtract
// per pair: (byte ^ 0x80) | 0x6400 is the fp16 value 1152 + c.  Q is
// converted to fp16 after multiplying each head by a power of two that puts
// its largest |q| in [2^14, 2^15) (exact, and undone in fp32 after the MMA).
// Because d is summed over, each thread owns a contiguous byte slice of every
// K row; Q's fragments use the same dim order.  The S accumulator fragment
// becomes the P operand fragment with one 8x8 transpose (movmatrix).
//
// The CTA merges its 4 warps' (m, l, O) and writes one partial per
// (sequence, q-head, split); decode_merge_kernel combines the splits,
// applies the epilogue and stores bf16.
#include "internal.h"

namespace fa {
namespace {

constexpr int kWarps = 4;
constexpr int kTile = 32;    // keys per tile
constexpr int kStages = 3;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const __nv_bfloat16* q;  // [B*hq, D]
  const float* k_scales;   // [B*hkv, cap]
  const float* v_scales;
  const int32_t* seqlens;  // [B]
  float* part_o;           // [B*hq, n_split_max, D]
  float* part_ml;          // [B*hq, n_split_max, 2]
  int hq, hkv, group, cap, window, split_keys, n_split_max, n_split_launched;
  float scale_log2;
  Watchdog wd;
};

template <int D>
struct Geom {
  static constexpr int kRowBytes = D;  // int8 codes
  static constexpr int kTileBytes = kTile * D;
  static constexpr int kScaleOff = 2 * kTileBytes;
  static constexpr int kStageBytes = ((2 * kTileBytes + 2 * kTile * 4) + 1023) / 1024 * 1024;
  static constexpr int kSwzMask = (D == 128) ? 0x70 : 0x30;  // 128B or 64B swizzle
  static constexpr int kSmem = kWarps * kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
};

// TMA swizzle of a byte offset inside a tile whose base is aligned to the
// swizzle period: bits [4,7) (128B) or [4,6) (64B) ^= bits [7,10) / [7,9).
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t lin) {
  return lin ^ ((lin >> 3) & Geom<D>::kSwzMask);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// fp16x2 of the signed bytes 0 and 2 of w (exact).
__device__ __forceinline__ uint32_t i8x2_to_f16x2_even(uint32_t w) {
  uint32_t t, r;
  asm("lop3.b32 %0, %1, 0x00ff00ff, 0x64806480, 0x6a;" : "=r"(t) : "r"(w));
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(0x64806480u));
  return r;
}
// fp16x2 of the signed bytes 1 and 3 of w (exact).
__device__ __forceinline__ uint32_t i8x2_to_f16x2_odd(uint32_t w) { return i8x2_to_f16x2_even(w >> 8); }

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Keys of sequence b handled by the decode: [k_lo, L); tiles start at the
// 32-aligned t_begin <= k_lo so every tile's scale block is 16-byte aligned.
__device__ __forceinline__ void key_range(int L, int window, int& k_lo, int& t_begin) {
  k_lo = window > 0 ? max(0, L - window) : 0;
  t_begin = (k_lo / kTile) * kTile;
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32, 2)
    decode_i8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecodeArgs A) {
  using G = Geom<D>;
  constexpr int kSteps = D / 16;      // k-steps of the S MMA
  constexpr int kChunks = D / 64;     // 16-byte chunks per thread per K row
  constexpr int kMT = D / 16;         // O^T m-tiles (dims)
  extern __shared__ uint8_t dec_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * G::kStageBytes);
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = max(0, min(A.seqlens[b], A.cap));
  int k_lo, t_begin;
  key_range(L, A.window, k_lo, t_begin);
  const int key_begin = t_begin + split * A.split_keys;
  if (key_begin >= L) return;
  const int key_end = min(L, key_begin + A.split_keys);
  const int n_tiles = (key_end - key_begin + kTile - 1) / kTile;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qq = lane & 3;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;
  const int64_t kv_row0 = (static_cast<int64_t>(b) * A.hkv + g) * A.cap;

  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[warp * kStages + s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto stage_ptr = [&](int s) { return smem + (warp * kStages + s) * G::kStageBytes; };
  auto issue = [&](int i) {  // tile i of this warp into stage i % kStages
    const int s = i % kStages;
    const int key0 = key_begin + (warp + i * kWarps) * kTile;
    uint8_t* st = stage_ptr(s);
    uint64_t* bar = &bars[warp * kStages + s];
    mbar_expect_tx(bar, 2 * G::kTileBytes + 2 * kTile * 4);
    tma_load_2d(st, &tm_k, bar, 0, static_cast<int>(kv_row0 + key0));
    tma_load_2d(st + G::kTileBytes, &tm_v, bar, 0, static_cast<int>(kv_row0 + key0));
    bulk_load(st + G::kScaleOff, A.k_scales + kv_row0 + key0, kTile * 4, bar);
    bulk_load(st + G::kScaleOff + kTile * 4, A.v_scales + kv_row0 + key0, kTile * 4, bar);
  };
  if (lane == 0) {
    for (int i = 0; i < min(kStages, my_tiles); ++i) issue(i);
  }

  // ---- Q fragments: thread (gq, qq) holds head gq, dims [qq*D/4, (qq+1)*D/4)
  uint32_t qb0[kSteps], qb1[kSteps];
  float qs_own = 0.f;
  {
    float qv[D / 4];
    const bool head_ok = gq < A.group;
    const int hq_idx = b * A.hq + g * A.group + gq;
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (head_ok) raw = *reinterpret_cast<const uint4*>(A.q + static_cast<int64_t>(hq_idx) * D + qq * (D / 4) + 8 * c);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
        qv[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < D / 4; ++e) amax = fmaxf(amax, fabsf(qv[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);
    const int kexp = amax > 0.f ? 15 - ex : 0;  // largest |q| * 2^kexp in [2^14, 2^15)
    qs_own = ldexpf(A.scale_log2, -kexp);
#pragma unroll
    for (int ks = 0; ks < kSteps; ++ks) {
      qb0[ks] = pack_f16x2(ldexpf(qv[4 * ks + 0], kexp), ldexpf(qv[4 * ks + 2], kexp));
      qb1[ks] = pack_f16x2(ldexpf(qv[4 * ks + 1], kexp), ldexpf(qv[4 * ks + 3], kexp));
    }
  }
  // logit multipliers of this thread's two score columns (heads 2qq, 2qq+1)
  const float qs0 = __shfl_sync(0xffffffffu, qs_own, (2 * qq) * 4);
  const float qs1 = __shfl_sync(0xffffffffu, qs_own, (2 * qq + 1) * 4);

  float o[kMT][4];
#pragma unroll
  for (int m = 0; m < kMT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int i = 0; i < my_tiles; ++i) {
    const int s = i % kStages;
    // every lane polls; the decision to continue is warp-uniform because the
    // MMAs and transposes below need the whole warp
    const bool ready = wait_parity(&bars[warp * kStages + s], (i / kStages) & 1, A.wd, &abort_flag);
    if (!__all_sync(0xffffffffu, ready)) break;
    const uint32_t kt = smem_u32(stage_ptr(s));
    const uint32_t vt = kt + G::kTileBytes;
    const float* ksc = reinterpret_cast<const float*>(stage_ptr(s) + G::kScaleOff);
    const float* vsc = ksc + kTile;
    const int key0 = key_begin + (warp + i * kWarps) * kTile;

    // ---- S^T = K . Q^T for the two 16-key halves of the tile
    float sc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
      const int r0 = 16 * mt + gq, r1 = r0 + 8;
      uint4 ka[kChunks], kb[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const uint32_t off = (qq * kChunks + c) * 16;
        ka[c] = lds128(kt + swz<D>(r0 * D + off));
        kb[c] = lds128(kt + swz<D>(r1 * D + off));
      }
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        const uint4& A4 = ka[ks / 4];
        const uint4& B4 = kb[ks / 4];
        const uint32_t wa = (ks % 4 == 0) ? A4.x : (ks % 4 == 1) ? A4.y : (ks % 4 == 2) ? A4.z : A4.w;
        const uint32_t wb = (ks % 4 == 0) ? B4.x : (ks % 4 == 1) ? B4.y : (ks % 4 == 2) ? B4.z : B4.w;
        mma16816(sc[mt], i8x2_to_f16x2_even(wa), i8x2_to_f16x2_even(wb), i8x2_to_f16x2_odd(wa),
                 i8x2_to_f16x2_odd(wb), qb0[ks], qb1[ks]);
      }
    }

    // ---- online softmax (per head column), masks by key position
    float x[2][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int kl = 16 * mt + gq + 8 * hf;
        const int key = key0 + kl;
        const bool ok = key >= k_lo && key < key_end;
        const float kscale = ksc[kl];
        x[mt][2 * hf + 0] = ok ? sc[mt][2 * hf + 0] * kscale * qs0 : -INFINITY;
        x[mt][2 * hf + 1] = ok ? sc[mt][2 * hf + 1] * kscale * qs1 : -INFINITY;
        mx0 = fmaxf(mx0, x[mt][2 * hf + 0]);
        mx1 = fmaxf(mx1, x[mt][2 * hf + 1]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2_approx(m_run[0] - ref0), al1 = ex2_approx(m_run[1] - ref1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    l_run[0] *= al0;
    l_run[1] *= al1;
#pragma unroll
    for (int m = 0; m < kMT; ++m) {
      o[m][0] *= al0; o[m][2] *= al0;
      o[m][1] *= al1; o[m][3] *= al1;
    }
    uint32_t pb[2][2];  // [mt][b0/b1] P' operand fragments
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t packed[2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int kl = 16 * mt + gq + 8 * hf;
        const int key = key0 + kl;
        const bool ok = key >= k_lo && key < key_end;
        const float p0 = ex2_approx(x[mt][2 * hf + 0] - ref0);
        const float p1 = ex2_approx(x[mt][2 * hf + 1] - ref1);
        l_run[0] += p0;
        l_run[1] += p1;
        const float vscale = ok ? vsc[kl] : 0.f;
        packed[hf] = pack_f16x2(ok ? p0 * vscale : 0.f, ok ? p1 * vscale : 0.f);
      }
      pb[mt][0] = transpose8x8(packed[0]);  // (head gq; keys 2qq, 2qq+1)
      pb[mt][1] = transpose8x8(packed[1]);  // (head gq; keys 8+2qq, 8+2qq+1)
    }

    // ---- O^T += V^T . P'
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int kk0 = 16 * mt + 2 * qq;
#pragma unroll
      for (int pr = 0; pr < D / 32; ++pr) {
        const uint32_t xw = (8 * pr + gq) * 4;  // byte offset of this thread's word
        const uint32_t w0 = lds32(vt + swz<D>((kk0 + 0) * D + xw));
        const uint32_t w1 = lds32(vt + swz<D>((kk0 + 1) * D + xw));
        const uint32_t w2 = lds32(vt + swz<D>((kk0 + 8) * D + xw));
        const uint32_t w3 = lds32(vt + swz<D>((kk0 + 9) * D + xw));
        const uint32_t t01l = prmt(w0, w1, 0x5410), t01h = prmt(w0, w1, 0x7632);
        const uint32_t t23l = prmt(w2, w3, 0x5410), t23h = prmt(w2, w3, 0x7632);
        mma16816(o[2 * pr], i8x2_to_f16x2_even(t01l), i8x2_to_f16x2_odd(t01l), i8x2_to_f16x2_even(t23l),
                 i8x2_to_f16x2_odd(t23l), pb[mt][0], pb[mt][1]);
        mma16816(o[2 * pr + 1], i8x2_to_f16x2_even(t01h), i8x2_to_f16x2_odd(t01h),
                 i8x2_to_f16x2_even(t23h), i8x2_to_f16x2_odd(t23h), pb[mt][0], pb[mt][1]);
      }
    }

    __syncwarp();
    if (lane == 0 && i + kStages < my_tiles) {
      fence_proxy_async_smem();
      issue(i + kStages);
    }
  }

  // ---- merge the 4 warps' states; then one partial per (q-head, split)
  l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 4);
  l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 4);
  l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 8);
  l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 8);
  l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 16);
  l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 16);
  __syncthreads();  // every warp is done with its stages (all issued tiles were waited on)
  float* red_o = reinterpret_cast<float*>(smem);          // [warp][8 heads][D]
  float* red_ml = red_o + kWarps * 8 * D;                  // [warp][8 heads][2]
  if (gq == 0) {
    red_ml[(warp * 8 + 2 * qq) * 2 + 0] = m_run[0];
    red_ml[(warp * 8 + 2 * qq) * 2 + 1] = l_run[0];
    red_ml[(warp * 8 + 2 * qq + 1) * 2 + 0] = m_run[1];
    red_ml[(warp * 8 + 2 * qq + 1) * 2 + 1] = l_run[1];
  }
#pragma unroll
  for (int pr = 0; pr < D / 32; ++pr) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int dim0 = 4 * (8 * pr + gq) + 2 * j;
      const float(&c)[4] = o[2 * pr + j];
      red_o[(warp * 8 + 2 * qq) * D + dim0] = c[0];
      red_o[(warp * 8 + 2 * qq + 1) * D + dim0] = c[1];
      red_o[(warp * 8 + 2 * qq) * D + dim0 + 1] = c[2];
      red_o[(warp * 8 + 2 * qq + 1) * D + dim0 + 1] = c[3];
    }
  }
  __syncthreads();
  const int active_warps = min(kWarps, n_tiles);
  for (int e = threadIdx.x; e < A.group * D; e += kWarps * 32) {
    const int h = e / D, dim = e % D;
    float M = -INFINITY;
    for (int w = 0; w < active_warps; ++w) M = fmaxf(M, red_ml[(w * 8 + h) * 2]);
    const float ref = M == -INFINITY ? 0.f : M;
    float acc = 0.f, lsum = 0.f;
    for (int w = 0; w < active_warps; ++w) {
      const float f = ex2_approx(red_ml[(w * 8 + h) * 2] - ref);
      acc += f * red_o[(w * 8 + h) * D + dim];
      lsum += f * red_ml[(w * 8 + h) * 2 + 1];
    }
    const int64_t rec = (static_cast<int64_t>(b) * A.hq + g * A.group + h) * A.n_split_max + split;
    A.part_o[rec * D + dim] = acc;
    if (dim == 0) {
      A.part_ml[rec * 2 + 0] = M;
      A.part_ml[rec * 2 + 1] = lsum;
    }
  }
}

// One CTA per (sequence, q-head): log-sum-exp merge of the split partials.
template <int D>
__global__ void __launch_bounds__(128)
    decode_merge_kernel(const DecodeArgs A, __nv_bfloat16* __restrict__ out, Epilogue epi) {
  const int bh = blockIdx.x;
  const int b = bh / A.hq;
  const int L = max(0, min(A.seqlens[b], A.cap));
  int k_lo, t_begin;
  key_range(L, A.window, k_lo, t_begin);
  const int n_split = min(A.n_split_launched, L > t_begin ? (L - t_begin + A.split_keys - 1) / A.split_keys : 0);
  const int64_t rec0 = static_cast<int64_t>(bh) * A.n_split_max;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, A.part_ml[(rec0 + s) * 2]);
  const float ref = M == -INFINITY ? 0.f : M;
  for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
    float acc = 0.f, lsum = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const float f = ex2_approx(A.part_ml[(rec0 + s) * 2] - ref);
      acc += f * A.part_o[(rec0 + s) * D + dim];
      lsum += f * A.part_ml[(rec0 + s) * 2 + 1];
    }
    const float y = lsum > 0.f ? acc / lsum : 0.f;
    out[static_cast<int64_t>(bh) * D + dim] = __float2bfloat16_rn(apply_epilogue(y, epi));
  }
}

template <int D>
fa_status launch_decode_i8(const fa_decode_params& p, int split_keys, int n_splits, const LaunchCtx& ctx) {
  using G = Geom<D>;
  const uint64_t rows = static_cast<uint64_t>(p.batch) * p.hkv * p.capacity;
  CUtensorMap tmk, tmv;
  const uint64_t dims[2] = {static_cast<uint64_t>(D), rows};
  const uint64_t strides[1] = {static_cast<uint64_t>(D)};
  const uint32_t box[2] = {static_cast<uint32_t>(D), static_cast<uint32_t>(kTile)};
  const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  fa_status st = encode_tensor_map(&tmk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p.k_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;
  st = encode_tensor_map(&tmv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p.v_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;

  const int n_split_max = (p.capacity + 255) / 256;
  const size_t o_bytes = static_cast<size_t>(p.batch) * p.hq * n_split_max * D * sizeof(float);
  DecodeArgs A;
  A.q = static_cast<const __nv_bfloat16*>(p.q);
  A.k_scales = p.k_scales;
  A.v_scales = p.v_scales;
  A.seqlens = p.cache_seqlens;
  A.part_o = static_cast<float*>(p.workspace);
  A.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(p.workspace) + o_bytes);
  A.hq = p.hq;
  A.hkv = p.hkv;
  A.group = p.hq / p.hkv;
  A.cap = p.capacity;
  A.window = p.window;
  A.split_keys = split_keys;
  A.n_split_max = n_split_max;
  A.n_split_launched = n_splits;
  A.scale_log2 = p.softmax_scale * kLog2e;
  A.wd = ctx.wd;

  auto kern = decode_i8_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem) != cudaSuccess)
    return FA_ERR_CUDA;
  note_variant(reinterpret_cast<const void*>(kern));
  dim3 grid(n_splits, p.hkv, p.batch);
  kern<<<grid, kWarps * 32, G::kSmem, ctx.stream>>>(tmk, tmv, A);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

  auto merge = decode_merge_kernel<D>;
  note_variant(reinterpret_cast<const void*>(merge));
  merge<<<p.batch * p.hq, 128, 0, ctx.stream>>>(A, static_cast<__nv_bfloat16*>(p.out),
                                                make_epilogue(p.epilogue, p.n_epilogue));
  return cuda_status(cudaGetLastError());
}

}  // namespace

fa_status launch_decode(const fa_decode_params& p, int split_keys, int n_splits, const LaunchCtx& ctx) {
  if (p.kv_dtype != FA_I8) return FA_ERR_UNSUPPORTED;
  if (p.head_dim == 128) return launch_decode_i8<128>(p, split_keys, n_splits, ctx);
  if (p.head_dim == 64) return launch_decode_i8<64>(p, split_keys, n_splits, ctx);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa

// ----------------------------------------------------------------------------
// Decode without caller workspace.
//
// For callers that cannot allocate device memory at call time -- for example
// a plug-in inside a serving runtime that owns every device byte through its
// own pre-planned arena and forbids allocations outside it, or a caller that
// must not risk the implicit device synchronisation a cudaMalloc can cause --
// the per-split partials (O, m, l) live in this file-scope device array
// instead of a caller workspace.  Every device that loads the library holds
// it until the process exits.  All calls on a device share it and it keeps
// the last call's contents; nothing in it needs clearing, because the merge
// only reads records that the same call's split kernel wrote.  Calls whose
// work overlaps on the GPU (different streams, or different host threads on
// the same device) race on the array and must be serialised by the caller.
#include <mutex>

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[kNoAllocScratchBytes];
// Watchdog word of this path (the library's shared status word is allocated
// lazily, which this path must not do).
static __device__ unsigned int g_decode_noalloc_status;

// Device addresses of the scratch array and status word for the current
// device.  The first call on each device looks them up (cudaGetSymbolAddress,
// with that device current); later calls reuse them.
fa_status noalloc_scratch(void** scratch, unsigned int** status) {
  static std::mutex mu;
  static void* addr[64] = {};
  static void* word[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    void* w = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    if (cudaGetSymbolAddress(&w, g_decode_noalloc_status) != cudaSuccess || w == nullptr) return FA_ERR_CUDA;
    word[dev] = w;
    addr[dev] = p;
  }
  *scratch = addr[dev];
  *status = static_cast<unsigned int*>(word[dev]);
  return FA_OK;
}

template <int D>
fa_status launch_decode_i8_noalloc(const fa_decode_params& p, int split_keys, int n_splits, void* scratch,
                                   const LaunchCtx& ctx) {
  using G = Geom<D>;
  const uint64_t rows = static_cast<uint64_t>(p.batch) * p.hkv * p.capacity;
  CUtensorMap tmk, tmv;
  const uint64_t dims[2] = {static_cast<uint64_t>(D), rows};
  const uint64_t strides[1] = {static_cast<uint64_t>(D)};
  const uint32_t box[2] = {static_cast<uint32_t>(D), static_cast<uint32_t>(kTile)};
  const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  fa_status st = encode_tensor_map(&tmk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p.k_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;
  st = encode_tensor_map(&tmv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p.v_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;

  // partial records are packed with a stride of the launched split count
  const size_t o_bytes = static_cast<size_t>(p.batch) * p.hq * n_splits * D * sizeof(float);
  DecodeArgs A;
  A.q = static_cast<const __nv_bfloat16*>(p.q);
  A.k_scales = p.k_scales;
  A.v_scales = p.v_scales;
  A.seqlens = p.cache_seqlens;
  A.part_o = static_cast<float*>(scratch);
  A.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + o_bytes);
  A.hq = p.hq;
  A.hkv = p.hkv;
  A.group = p.hq / p.hkv;
  A.cap = p.capacity;
  A.window = p.window;
  A.split_keys = split_keys;
  A.n_split_max = n_splits;
  A.n_split_launched = n_splits;
  A.scale_log2 = p.softmax_scale * kLog2e;
  A.wd = ctx.wd;

  auto kern = decode_i8_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem) != cudaSuccess)
    return FA_ERR_CUDA;
  // (no note_variant here: its bookkeeping set may allocate host memory)
  dim3 grid(n_splits, p.hkv, p.batch);
  kern<<<grid, kWarps * 32, G::kSmem, ctx.stream>>>(tmk, tmv, A);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  auto merge = decode_merge_kernel<D>;
  merge<<<p.batch * p.hq, 128, 0, ctx.stream>>>(A, static_cast<__nv_bfloat16*>(p.out),
                                                make_epilogue(p.epilogue, p.n_epilogue));
  return cuda_status(cudaGetLastError());
}

}  // namespace

size_t decode_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

fa_status launch_decode_noalloc(const fa_decode_params& p, int split_keys, long long budget, cudaStream_t stream) {
  if (p.kv_dtype != FA_I8) return FA_ERR_UNSUPPORTED;
  const int max_len = p.max_seqlen > 0 ? p.max_seqlen : p.capacity;
  const size_t per_split = static_cast<size_t>(p.batch) * p.hq * (p.head_dim + 2) * sizeof(float);
  if (per_split > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;  // even one split does not fit
  const int fit = static_cast<int>(kNoAllocScratchBytes / per_split);
  int n_splits = max_len > 0 ? (max_len + split_keys - 1) / split_keys : 1;
  if (n_splits > fit) {
    if (p.split_keys > 0) return FA_ERR_WORKSPACE;  // the caller's split count does not fit
    split_keys = ((max_len + fit - 1) / fit + 255) / 256 * 256;
    n_splits = (max_len + split_keys - 1) / split_keys;
    if (n_splits > fit) return FA_ERR_WORKSPACE;
  }
  if (n_splits < 1) n_splits = 1;
  void* scratch = nullptr;
  LaunchCtx ctx;
  ctx.stream = stream;
  ctx.wd.budget = budget;
  fa_status st = noalloc_scratch(&scratch, &ctx.wd.word);
  if (st != FA_OK) return st;
  if (p.head_dim == 128) return launch_decode_i8_noalloc<128>(p, split_keys, n_splits, scratch, ctx);
  if (p.head_dim == 64) return launch_decode_i8_noalloc<64>(p, split_keys, n_splits, scratch, ctx);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
