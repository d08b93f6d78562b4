// prefill_tc.cu -- fused attention forward on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), bf16 Q/K/V, fp32 accumulation.
//
// What it computes: fkl_python PR #6, Summary -- FlashAttention-2 style
// forward softmax(q k^T * scale + mask) v with fused epilogue ops, layout
// (batch*heads, seq, head_dim) or varlen; online softmax rescaling (Foundry
// attention/README.md, References: the FlashAttention paper and the online
// softmax trick), so the score matrix never leaves the SM.
//
// Persistent CTAs (one per SM) walk work items in longest-first order; the
// next item's Q, first K/V tiles and first S MMAs run under the current
// item's last softmax, PV and epilogue (its Q is reloaded once the current
// item's S MMAs have read it, its first PV waits until O has been read out).
//
// CTA work tile: two 128-row Q tiles = the same 128 query rows of two query
// heads of one GQA group (SKaiNET-transformers PR #419, Summary: one task per
// GQA group).  Both tiles see the same mask, so they walk the same key range
// and every K/V tile brought in by TMA serves both heads.  (An odd group
// size runs one Q tile per CTA.)  Key tiles outside the causal / window band
// are never loaded; only boundary tiles get an element mask.
//
// Warp roles (320 threads):
//   warps 0-3  softmax of Q tile 0 (one thread per row = one TMEM lane)
//   warps 4-7  softmax of Q tile 1
//   warp 8     TMA producer: Q once, then a K ring and a V ring
//   warp 9     MMA issuer (one thread) and TMEM owner
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
// P (bf16, two per 32-bit column) overwrites the first 64 columns of its S
// tile and is the A operand of O += P V straight from TMEM.
//
// Result modes: the normalised output (epilogue applied, bf16); that output
// with each row's log-sum-exp (a partial result over the given keys); or,
// for a result built up over several key blocks (the ring steps of a
// context-parallel prefill -- kernbench2 commit message, ADR-0060 (long
// context): an online-softmax merge at every ring step), merged in the
// epilogue into an fp32 accumulator (o, lse) that the softmax warps
// prefetch into L2 when an item starts, so no separate merge pass runs.
//
// MMA issue order per key tile j (ping-pong between the two Q tiles):
//   PV0(j-1), S0(j), PV1(j-1), S1(j)
// so the tensor core works on one tile while the other tile's softmax runs.
// Softmax of tile t at step j: wait S_t(j) (its commit also covers PV_t(j-1)),
// read the row, raise the running max only when it grows by more than 8 (in
// log2 units; the final O / l uses the same stale max, so the result is
// exact), rescale O_t in TMEM when it did, write P_t, signal the MMA warp.
// Every wait is bounded (device.cuh); a timeout aborts all roles cleanly.
//
// int8 K/V (fkl_python PR #6, Summary: the fused kernel dequantises on chip
// for both products and never widens the cache in global memory): TMA
// brings each int8 tile into shared memory (at d = 128 into the upper half of
// the bf16 slot it becomes); four converter warps, one thread per key row,
// dequantise it as c * s in fp32 (exact: |c| <= 127 times an fp32 scale),
// round once to bf16, the tensor-core operand type, write it in the operand
// layout and fence it to the async proxy.  The softmax is then the bf16 one.
// That variant runs 16 warps and rebalances registers with setmaxnreg
// (softmax 192, the rest 64).
#include "internal.h"
#include "layout.cuh"
#include "umma.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per Q tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp0 = 12;  // int8 variant: warps 12-15 convert K/V tiles
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kChunkBytes = kSwizzleChunkRows * 128;  // [128 rows x 64 bf16]

template <int D, bool kI8>
struct TcGeom {
  // K is consumed one step before V (S(j) precedes PV(j)), so K gets the
  // deeper ring: a slot refills with the TMA latency hidden behind ~2 steps
  static constexpr int kKStages = 3;
  static constexpr int kVStages = (D == 128) ? 2 : 3;
  static constexpr uint32_t kQBytes = kBM * D * 2;
  static constexpr uint32_t kKVBytes = kBN * D * 2;   // one bf16 K or V tile
  static constexpr uint32_t kI8Bytes = kBN * D;       // one int8 tile
  static constexpr uint32_t kKOff = 2 * kQBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kKVBytes;
  // int8 staging: at d = 128 in the upper half of each bf16 slot (a row's
  // bf16 output overwrites only that row's int8 bytes); at d = 64 separate
  static constexpr bool kInPlace = (D == 128);
  static constexpr uint32_t kStageOff = kVOff + kVStages * kKVBytes;
  static constexpr uint32_t kStageBytes = (kI8 && !kInPlace) ? (kKStages + kVStages) * kI8Bytes : 0;
  static constexpr uint32_t kBarOff = kStageOff + kStageBytes;
  static constexpr uint32_t kSmem = kBarOff + 256 + 1024;
  static constexpr int kThreads = kI8 ? 512 : 320;
  __host__ __device__ static constexpr uint32_t k_stage(int s) {
    return kInPlace ? kKOff + s * kKVBytes + kKVBytes / 2 : kStageOff + s * kI8Bytes;
  }
  __host__ __device__ static constexpr uint32_t v_stage(int s) {
    return kInPlace ? kVOff + s * kKVBytes + kKVBytes / 2 : kStageOff + (kKStages + s) * kI8Bytes;
  }
};
static_assert(TcGeom<128, false>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<128, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<64, true>::kSmem <= 232448, "shared memory budget");

struct PrefillArgs {
  SeqLayout L;
  __nv_bfloat16* out;
  float* lse;  // optional [rows of out]: log-sum-exp of the scaled scores (partial results)
  float* acc_o;    // optional fp32 [rows of out, D] accumulator merged into (with acc_lse)
  float* acc_lse;
  int acc_first;   // the accumulator holds nothing yet: not read
  int acc_last;    // merged rows go to out (epilogue applied); the accumulator is not written
  const float* k_scales;  // int8 variant: one fp32 scale per K / V row
  const float* v_scales;
  int64_t k_plane_rows;   // rows per K plane (the scales share K's row numbering)
  int batch, hq, hkv, group, n_qblocks, two_tiles;
  float scale_log2;      // |softmax scale| * log2(e), > 0
  uint32_t negate_s;     // 1: the MMA negates Q (a negative softmax scale)
  Epilogue epi;
  Watchdog wd;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Four signed bytes of w times the row scale, each product rounded once to
// bf16 (two bf16x2 words).  Each byte b, flipped to b ^ 0x80 = c + 128, is
// placed in the low mantissa byte of 2^23, so the float is 2^23 + 128 + c and
// one exact subtraction leaves c; c * s is then exact in fp32 (8 x 24 bits
// fit), and the bf16 cast is the only rounding.
__device__ __forceinline__ uint2 dequant4_bf16(uint32_t w, float2 s2) {
  const uint32_t x = w ^ 0x80808080u;
  uint32_t f[4];
  asm("prmt.b32 %0, %1, 0x4b000000, 0x7540;" : "=r"(f[0]) : "r"(x));
  asm("prmt.b32 %0, %1, 0x4b000000, 0x7541;" : "=r"(f[1]) : "r"(x));
  asm("prmt.b32 %0, %1, 0x4b000000, 0x7542;" : "=r"(f[2]) : "r"(x));
  asm("prmt.b32 %0, %1, 0x4b000000, 0x7543;" : "=r"(f[3]) : "r"(x));
  const float2 bias = make_float2(-8388736.f, -8388736.f);  // -(2^23 + 128)
  const float2 c01 = add2(make_float2(__uint_as_float(f[0]), __uint_as_float(f[1])), bias);
  const float2 c23 = add2(make_float2(__uint_as_float(f[2]), __uint_as_float(f[3])), bias);
  const float2 y01 = mul2(c01, s2), y23 = mul2(c23, s2);
  return make_uint2(pack_bf16x2(y01.x, y01.y), pack_bf16x2(y23.x, y23.y));
}

// One work item: 128 query rows of one head pair (or one head), in the
// longest-first order (highest q-block first, then sequence, then head pair).
struct Item {
  Seq sq;
  int b, h0, g, i0, j_lo, n_iter;
  int q_plane, q_prow, k_plane, k_prow0;  // TMA coordinates
};
// False for an item with no row or no visible key (the empty-band kernel
// writes such rows).
__device__ __forceinline__ bool item_of(const PrefillArgs& A, int item, Item& w) {
  const int n_pairs = A.two_tiles ? A.hq / 2 : A.hq;
  const int per_qb = A.batch * n_pairs;
  const int qb = A.n_qblocks - 1 - item / per_qb;
  const int rem = item % per_qb;
  w.b = rem / n_pairs;
  const int pair = rem % n_pairs;
  w.h0 = A.two_tiles ? 2 * pair : pair;
  w.g = w.h0 / A.group;
  w.sq = seq_of(A.L, w.b, w.h0, w.g);
  w.i0 = qb * kBM;
  if (w.i0 >= w.sq.s_q) return false;
  const int i_last = min(w.i0 + kBM, w.sq.s_q) - 1;
  int lo_first, hi_first, lo_last, hi_last;
  band_of(A.L, w.i0, w.sq.s_q, w.sq.s_k, lo_first, hi_first);
  band_of(A.L, i_last, w.sq.s_q, w.sq.s_k, lo_last, hi_last);
  const int k_lo = max(0, lo_first);
  const int k_hi = min(w.sq.s_k, hi_last);
  w.j_lo = k_lo / kBN;
  w.n_iter = k_hi > k_lo ? (k_hi + kBN - 1) / kBN - w.j_lo : 0;
  if (w.n_iter == 0) return false;
  // dense planes are (b*h + h), varlen planes are h with the sequence
  // starting at cu[b] inside the plane
  const bool varlen = A.L.cu_q != nullptr;
  w.q_plane = varlen ? w.h0 : w.b * A.hq + w.h0;
  w.q_prow = (varlen ? A.L.cu_q[w.b] : 0) + w.i0;
  w.k_plane = varlen ? w.g : w.b * A.hkv + w.g;
  w.k_prow0 = varlen ? A.L.cu_k[w.b] : 0;
  return true;
}

// TMA plane and row of the 128-key tile starting at key0 of item w (paged:
// through the block table; a page id outside the pool reads page 0 and is
// reported).
__device__ __forceinline__ void kv_tile(const PrefillArgs& A, const Item& w, int key0, int& plane, int& row) {
  if (A.L.block_table == nullptr) {
    plane = w.k_plane;
    row = w.k_prow0 + key0;
    return;
  }
  bool bad;
  paged_key(A.L, w.b, w.g, key0, plane, row, bad);
  if (bad) record_status(A.wd, kStatusRange);
}

// The k-th item of CTA c among G persistent CTAs: rounds of G items in the
// longest-first order, walked forwards in even rounds and backwards in odd
// ones, so each CTA's total stays close to the others' (a plain stride gives
// CTA 0 the longest item of every round).
__device__ __forceinline__ int item_at(int c, int G, int k) {
  const int round = k, base = round * G;
  return (round & 1) ? base + (G - 1 - c) : base + c;
}

template <int D, bool kI8>
__global__ void __launch_bounds__(TcGeom<D, kI8>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillArgs A) {
  using G = TcGeom<D, kI8>;
  constexpr int KS = G::kKStages, VS = G::kVStages;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;  // [2]
  uint64_t* p_full = s_full + 2;   // [2 tiles][2 halves of the keys]
  uint64_t* o_done = p_full + 4;   // [2]
  uint64_t* drain = o_done + 2;
  uint64_t* kraw_full = drain + 1;   // [KS] int8 variant: TMA landed the int8 K tile
  uint64_t* vraw_full = kraw_full + KS;
  uint64_t* q_empty = vraw_full + VS;  // every S MMA of an item has read Q
  uint64_t* o_free = q_empty + 1;       // [2] the softmax warps have read O_t out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_free + 2);
  __shared__ int abort_flag;

  // Persistent CTAs: CTA c takes one item per round of gridDim.x items of the
  // longest-first order (item_at); every role walks the same sequence, with
  // the K/V ring and every barrier phase counted across items.
  const int n_items = A.n_qblocks * A.batch * (A.two_tiles ? A.hq / 2 : A.hq);
  const int ntile = A.two_tiles ? 2 : 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    // bf16: TMA completes k_full / v_full; int8: the 128 converter threads do
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, kI8 ? 128 : 1);
      mbar_init(k_empty + s, 1);
      mbar_init(kraw_full + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, kI8 ? 128 : 1);
      mbar_init(v_empty + s, 1);
      mbar_init(vraw_full + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + 2 * t, kBM);
      mbar_init(p_full + 2 * t + 1, kBM);
      mbar_init(o_done + t, 1);
    }
    mbar_init(drain, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_free, kBM);
    mbar_init(o_free + 1, kBM);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Roles split by warpgroup first: warpgroups 0-1 softmax, 2-3 the rest.
  // int8 variant registers: 512 threads launched at 128; warpgroups 0-1 take
  // 192, warpgroups 2-3 give back down to 64: 256*192 + 256*64 = 512*128.
  if (warp >= 8) {
  if constexpr (kI8) asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      int base = 0, done = 0;  // K/V tiles and items before this one
      bool ok = true;
      for (int k = 0, item; ok && (item = item_at(blockIdx.x, gridDim.x, k)) < n_items; ++k) {
        Item w;
        if (!item_of(A, item, w)) continue;
        // Q of this item once every S MMA of the previous one has read its Q
        if (done > 0 && !wait_parity(q_empty, (done - 1) & 1, A.wd, &abort_flag)) break;
        mbar_expect_tx(q_full, ntile * G::kQBytes);
        for (int t = 0; t < ntile; ++t)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + t * G::kQBytes + c * kChunkBytes, &tm_q, q_full, 64 * c, w.q_prow, w.q_plane + t);
        for (int it = 0; it < w.n_iter; ++it) {
          const int gi = base + it;
          int s = gi % KS, u = gi / KS;
          int kplane, krow;
          kv_tile(A, w, (w.j_lo + it) * kBN, kplane, krow);
          if (u > 0 && !(ok = wait_parity(k_empty + s, (u - 1) & 1, A.wd, &abort_flag))) break;
          if constexpr (kI8) {
            mbar_expect_tx(kraw_full + s, G::kI8Bytes);
            tma_load_3d(smem + G::k_stage(s), &tm_k, kraw_full + s, 0, krow, kplane);
          } else {
            mbar_expect_tx(k_full + s, G::kKVBytes);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + G::kKOff + s * G::kKVBytes + c * kChunkBytes, &tm_k, k_full + s, 64 * c, krow,
                          kplane);
          }
          s = gi % VS;
          u = gi / VS;
          if (u > 0 && !(ok = wait_parity(v_empty + s, (u - 1) & 1, A.wd, &abort_flag))) break;
          if constexpr (kI8) {
            mbar_expect_tx(vraw_full + s, G::kI8Bytes);
            tma_load_3d(smem + G::v_stage(s), &tm_v, vraw_full + s, 0, krow, kplane);
          } else {
            mbar_expect_tx(v_full + s, G::kKVBytes);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + G::kVOff + s * G::kKVBytes + c * kChunkBytes, &tm_v, v_full + s, 64 * c, krow,
                          kplane);
          }
        }
        base += w.n_iter;
        ++done;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // a negative softmax scale is folded into the S MMA (negated A operand),
      // so the softmax only ever sees a positive scale
      const uint32_t idesc_s = umma_idesc_f16(kBM, kBN, 1, 1, false) | (A.negate_s << 13);
      constexpr uint32_t idesc_o = umma_idesc_f16(kBM, D, 1, 1, true);
      const uint32_t q_base = smem_u32(smem);
      // operand descriptors are built once; a k-step only moves the start
      // address (its 14-bit field never carries: every address is < 2^18)
      const uint64_t dq0 = umma_desc_sw128(q_base, 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(q_base + G::kKOff, 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(q_base + G::kVOff, kChunkBytes, 1024);
      auto issue_s = [&](int t, int st) {
        const uint64_t dq = dq0 + ((t * G::kQBytes) >> 4);
        const uint64_t dk = dk0 + ((st * G::kKVBytes) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k / 4) * kChunkBytes + (k % 4) * 32) >> 4;
          mma_ss(tmem + t * kBN, dq + off, dk + off, idesc_s, k > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V over keys [64 h, 64 h + 64)
      auto issue_pv_half = [&](int t, int st, int h, bool accumulate) {
        const uint64_t dv = dv0 + ((st * G::kKVBytes) >> 4);
#pragma unroll
        for (int k = 4 * h; k < 4 * h + 4; ++k) {
          mma_ts(tmem + 256 + t * D, tmem + t * kBN + k * 8, dv + ((k * 2048) >> 4), idesc_o,
                 (accumulate || k > 0) ? 1u : 0u);
        }
      };
      int base = 0, done = 0;  // K/V tiles and items before the current one
      // PV for step j (of the current item) of tile t, each half as soon as
      // the softmax wrote it; an item's first PV overwrites O_t, so it also
      // waits until the previous item's O_t has been read out
      auto issue_pv = [&](int t, int j) -> bool {
        const int gj = base + j;
        const int vs = gj % VS;
        if (j == 0 && done > 0 && !wait_parity(o_free + t, (done - 1) & 1, A.wd, &abort_flag)) return false;
        if (!wait_parity(p_full + 2 * t, gj & 1, A.wd, &abort_flag)) return false;
        if (t == 0 && !wait_parity(v_full + vs, (gj / VS) & 1, A.wd, &abort_flag)) return false;
        tc_fence_after();
        issue_pv_half(t, vs, 0, j > 0);
        if (!wait_parity(p_full + 2 * t + 1, gj & 1, A.wd, &abort_flag)) return false;
        tc_fence_after();
        issue_pv_half(t, vs, 1, true);
        return true;
      };
      bool ok = true;
      for (int k = 0, item; ok && (item = item_at(blockIdx.x, gridDim.x, k)) < n_items; ++k) {
        Item w;
        if (!item_of(A, item, w)) continue;
        if (!(ok = wait_parity(q_full, done & 1, A.wd, &abort_flag))) break;
        for (int it = 0; ok && it < w.n_iter; ++it) {
          const int gi = base + it;
          const int s = gi % KS;
          if (!(ok = wait_parity(k_full + s, (gi / KS) & 1, A.wd, &abort_flag))) break;
          tc_fence_after();
          for (int t = 0; t < ntile; ++t) {
            if (it > 0) {
              if (!(ok = issue_pv(t, it - 1))) break;
              if (t == ntile - 1) mma_commit(v_empty + (gi - 1) % VS);
            }
            issue_s(t, s);
            mma_commit(s_full + t);
          }
          if (ok) mma_commit(k_empty + s);
        }
        if (!ok) break;
        mma_commit(q_empty);  // Q is free once this item's S MMAs complete
        for (int t = 0; t < ntile; ++t) {
          if (!(ok = issue_pv(t, w.n_iter - 1))) break;
          mma_commit(o_done + t);
        }
        if (!ok) break;
        mma_commit(v_empty + (base + w.n_iter - 1) % VS);
        base += w.n_iter;
        ++done;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(drain);
      wait_parity(drain, 0, A.wd);
    }
  } else if (kI8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ int8 -> bf16 converters
    // thread r rewrites row r of each int8 K and V tile as bf16 in the
    // 128-byte-swizzled K-major (K) / MN-major (V) operand layout
    const int r = static_cast<int>(threadIdx.x) - kConvWarp0 * 32;
    auto convert_row = [&](const uint8_t* src_tile, uint8_t* dst_tile, float sc) {
      const float2 s2 = make_float2(sc, sc);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {  // 16-byte int8 chunks of the row
        const int pc = (D == 128) ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
        const uint4 w = *reinterpret_cast<const uint4*>(src_tile + r * D + pc * 16);
        const int h = c / 4, j0 = 2 * (c % 4);
        uint8_t* row = dst_tile + h * kChunkBytes + r * 128;
        const uint2 y0 = dequant4_bf16(w.x, s2), y1 = dequant4_bf16(w.y, s2);
        const uint2 y2 = dequant4_bf16(w.z, s2), y3 = dequant4_bf16(w.w, s2);
        *reinterpret_cast<uint4*>(row + ((j0 ^ (r & 7)) * 16)) = make_uint4(y0.x, y0.y, y1.x, y1.y);
        *reinterpret_cast<uint4*>(row + (((j0 + 1) ^ (r & 7)) * 16)) = make_uint4(y2.x, y2.y, y3.x, y3.y);
      }
    };
    int base = 0;
    bool ok = true;
    for (int k = 0, item; ok && (item = item_at(blockIdx.x, gridDim.x, k)) < n_items; ++k) {
      Item w;
      if (!item_of(A, item, w)) continue;
      for (int it = 0; it < w.n_iter; ++it) {
        const int gi = base + it;
        const int s = gi % KS, sv = gi % VS;
        const uint32_t ph = (gi / KS) & 1, phv = (gi / VS) & 1;
        // this thread's key row: its two scales, loaded ahead of the waits (0
        // past the sequence end, so those rows become zeros; the softmax masks them)
        const int key0 = (w.j_lo + it) * kBN;
        float ksc = 0.f, vsc = 0.f;
        if (key0 + r < w.sq.s_k) {
          int kplane, krow;
          kv_tile(A, w, key0, kplane, krow);
          const int64_t at = static_cast<int64_t>(kplane) * A.k_plane_rows + krow + r;
          ksc = __ldg(A.k_scales + at);
          vsc = __ldg(A.v_scales + at);
        }
        if (!(ok = __all_sync(0xffffffffu, wait_parity(kraw_full + s, ph, A.wd, &abort_flag)))) break;
        convert_row(smem + G::k_stage(s), smem + G::kKOff + s * G::kKVBytes, ksc);
        fence_proxy_async_smem();
        mbar_arrive(k_full + s);
        if (!(ok = __all_sync(0xffffffffu, wait_parity(vraw_full + sv, phv, A.wd, &abort_flag)))) break;
        convert_row(smem + G::v_stage(sv), smem + G::kVOff + sv * G::kKVBytes, vsc);
        fence_proxy_async_smem();
        mbar_arrive(v_full + sv);
      }
      base += w.n_iter;
    }
  }
  } else {
  if constexpr (kI8) asm volatile("setmaxnreg.inc.sync.aligned.u32 192;" ::: "memory");
  if (warp / 4 < ntile) {
    // ------------------------------------------------------------ softmax
    const int t = warp / 4, quarter = warp % 4;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + t * kBN;
    const uint32_t o_tm = tmem + lane_base + 256 + t * D;
    int base = 0, done = 0;  // K/V tiles and items before the current one
    bool ok = true;
    for (int k = 0, item; ok && (item = item_at(blockIdx.x, gridDim.x, k)) < n_items; ++k) {
    Item w;
    if (!item_of(A, item, w)) continue;
    const int i = w.i0 + r;
    int lo, hi;
    band_of(A.L, i, w.sq.s_q, w.sq.s_k, lo, hi);
    const int64_t out_row = w.sq.q_row0 + static_cast<int64_t>(t) * A.L.q_hstride + i;
    if (A.acc_o != nullptr && !A.acc_first && i < w.sq.s_q) {
      // the accumulator row is read in this item's epilogue: start it towards L2
      const char* arow = reinterpret_cast<const char*>(A.acc_o + out_row * D);
#pragma unroll
      for (int c = 0; c < D * 4; c += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(arow + c));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(A.acc_lse + out_row));
    }
    float m_used = -INFINITY, l = 0.f;
    for (int it = 0; it < w.n_iter; ++it) {
      ok = __all_sync(0xffffffffu, wait_parity(s_full + t, (base + it) & 1, A.wd, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t raw[4][32];
      tmem_ld32(s_tm + 0, raw[0]);
      tmem_ld32(s_tm + 32, raw[1]);
      tmem_ld32(s_tm + 64, raw[2]);
      tmem_ld32(s_tm + 96, raw[3]);
      tmem_wait_ld();
      const int kb = (w.j_lo + it) * kBN;
      if (!(kb >= lo && kb + kBN <= hi)) {
        // boundary tile: keys outside this row's band become -inf (the
        // softmax scale is positive, so masking before it is the same)
        const int va = lo - kb, vb = hi - kb;
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c < va || c >= vb) raw[c / 32][c % 32] = 0xff800000u;
      }
      // row max of the raw scores: eight independent chains of 3-input max
      float g8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t* v = &raw[k / 2][(k % 2) * 16];
        float g = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int e = 3; e < 15; e += 2) g = max3f(g, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        g8[k] = fmaxf(g, __uint_as_float(v[15]));
      }
      const float m_raw = fmaxf(max3f(g8[0], g8[1], g8[2]), max3f(max3f(g8[3], g8[4], g8[5]), g8[6], g8[7]));
      const float m_tile = m_raw * A.scale_log2;
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const float2 sc2 = make_float2(A.scale_log2, A.scale_log2);
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 lacc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) lacc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // p = 2^(s * scale * log2(e) - m): one packed FMA for two scores
          const float2 x = fma2(make_float2(__uint_as_float(raw[cc][2 * e]), __uint_as_float(raw[cc][2 * e + 1])),
                                sc2, nm2);
          const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          lacc[e % 8] = add2(lacc[e % 8], pp);
          pk[e] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st16(s_tm + cc * 16, pk);
        if (cc == 1 && it > 0 && __any_sync(0xffffffffu, need)) {
          // O_t is idle here (PV_t of the previous step has completed, this
          // step's starts only after the signal below): rescale it if some
          // row's max moved (rare; the first half's scores are dead by now)
#pragma unroll
          for (int oc = 0; oc < D / 32; ++oc) {
            uint32_t o[32];
            tmem_ld32(o_tm + oc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(o_tm + oc * 32, o);
          }
        }
        if (cc % 2 == 1) {
          // keys [64 h, 64 h + 64) of P are in TMEM: let the PV MMA start on them
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full + 2 * t + cc / 2);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) lacc[k] = add2(lacc[k], lacc[k + 4]);
      lacc[0] = add2(lacc[0], lacc[2]);
      lacc[1] = add2(lacc[1], lacc[3]);
      lacc[0] = add2(lacc[0], lacc[1]);
      l = l * alpha + (lacc[0].x + lacc[0].y);
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_parity(o_done + t, done & 1, A.wd, &abort_flag));
    if (!ok) break;
    tc_fence_after();
    const bool has_keys = lo < hi;
    const bool acc = A.acc_o != nullptr;
    // with lse (partial results) a row without keys is the epilogue of 0 with
    // lse = -inf; otherwise (and always when accumulating) the empty-band
    // kernel writes it
    const bool store = i < w.sq.s_q && (has_keys || (A.lse != nullptr && !acc));
    float inv_l = has_keys ? 1.f / l : 0.f;
    float w_acc = 0.f;  // accumulate mode: o_new = w_acc * o_acc + inv_l * O
    if (store && (A.lse != nullptr || acc)) {
      const float lse_part = has_keys ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      if (A.lse != nullptr) A.lse[out_row] = lse_part;
      if (acc) {
        // merge by log-sum-exp: lse = log(e^lse_acc + e^lse_part), each side
        // weighted by e^(its lse - lse); this row has keys, so lse_part is finite
        const float la = A.acc_first ? -INFINITY : A.acc_lse[out_row];
        const float mx = fmaxf(la, lse_part);
        const float ea = expf(la - mx), eb = expf(lse_part - mx), sum = ea + eb;
        w_acc = ea / sum;
        inv_l *= eb / sum;
        if (!A.acc_last) A.acc_lse[out_row] = mx + logf(sum);
      }
    }
    __nv_bfloat16* orow = A.out != nullptr ? A.out + out_row * D : nullptr;
    float* arow = acc ? A.acc_o + out_row * D : nullptr;
#pragma unroll
    for (int oc = 0; oc < D / 32; ++oc) {
      uint32_t o[32];
      tmem_ld32(o_tm + oc * 32, o);
      tmem_wait_ld();
      if (oc == D / 32 - 1) {
        // O_t is in registers: the next item's first PV may overwrite it
        tc_fence_before();
        mbar_arrive(o_free + t);
      }
      float y[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(o[e]) * inv_l;
      if (acc && store && w_acc != 0.f) {
        const float4* src = reinterpret_cast<const float4*>(arow + oc * 32);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 a = src[v];
          y[4 * v] = fmaf(a.x, w_acc, y[4 * v]);
          y[4 * v + 1] = fmaf(a.y, w_acc, y[4 * v + 1]);
          y[4 * v + 2] = fmaf(a.z, w_acc, y[4 * v + 2]);
          y[4 * v + 3] = fmaf(a.w, w_acc, y[4 * v + 3]);
        }
      }
      if (acc && !A.acc_last) {
        if (store) {
          float4* dst = reinterpret_cast<float4*>(arow + oc * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v) dst[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
        }
        continue;
      }
      apply_epilogue_vec(y, A.epi);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow + oc * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    base += w.n_iter;
    ++done;
    }
  }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool kI8>
fa_status launch_tc(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink, const LaunchCtx& ctx) {
  using G = TcGeom<D, kI8>;
  const bool varlen = p.cu_seqlens_q != nullptr;
  const uint64_t q_rows = varlen ? p.total_q : p.seqlen_q;
  // paged keys: planes of page_size rows, one per (page, KV head)
  const uint64_t k_rows = pages != nullptr ? pages->page_size : (varlen ? p.total_k : p.seqlen_k);
  const uint64_t q_planes = varlen ? p.hq : static_cast<uint64_t>(p.batch) * p.hq;
  const uint64_t k_planes = pages != nullptr ? static_cast<uint64_t>(pages->num_pages) * p.hkv
                                             : (varlen ? p.hkv : static_cast<uint64_t>(p.batch) * p.hkv);
  if (k_rows == 0) return FA_OK;  // no keys anywhere: only the empty-band kernel writes
  CUtensorMap tq, tk, tv;
  {
    const uint32_t box[3] = {64, static_cast<uint32_t>(kSwizzleChunkRows), 1};
    const uint64_t dims[3] = {static_cast<uint64_t>(D), q_rows, q_planes};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, q_rows * D * 2};
    fa_status st = encode_tensor_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.q, dims, strides, box,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }
  if constexpr (kI8) {
    // int8 rows of D bytes, one box per tile (128 B or 64 B swizzle)
    const uint32_t box[3] = {static_cast<uint32_t>(D), static_cast<uint32_t>(kSwizzleChunkRows), 1};
    const uint64_t dims[3] = {static_cast<uint64_t>(D), k_rows, k_planes};
    const uint64_t strides[2] = {static_cast<uint64_t>(D), k_rows * D};
    const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    fa_status st = encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p.k, dims, strides, box, sw);
    if (st != FA_OK) return st;
    st = encode_tensor_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p.v, dims, strides, box, sw);
    if (st != FA_OK) return st;
  } else {
    const uint32_t box[3] = {64, static_cast<uint32_t>(kSwizzleChunkRows), 1};
    const uint64_t dims[3] = {static_cast<uint64_t>(D), k_rows, k_planes};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, k_rows * D * 2};
    fa_status st = encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.k, dims, strides, box,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
    st = encode_tensor_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.v, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }
  PrefillArgs A;
  A.L = pages != nullptr ? SeqLayout::paged(p, *pages) : SeqLayout::from(p);
  A.out = static_cast<__nv_bfloat16*>(p.out);
  A.lse = sink.lse;
  A.acc_o = sink.acc_o;
  A.acc_lse = sink.acc_lse;
  A.acc_first = sink.first;
  A.acc_last = sink.last;
  A.k_scales = p.k_scales;
  A.v_scales = p.v_scales;
  A.k_plane_rows = static_cast<int64_t>(k_rows);
  A.batch = p.batch;
  A.hq = p.hq;
  A.hkv = p.hkv;
  A.group = p.hq / p.hkv;
  A.two_tiles = (A.group % 2 == 0) ? 1 : 0;
  const int max_sq = varlen ? p.max_seqlen_q : p.seqlen_q;
  A.n_qblocks = (max_sq + kBM - 1) / kBM;
  // the softmax works with a positive scale: a negative one negates Q inside
  // the S MMA; a zero scale (uniform weights) becomes a vanishing one
  const float abs_scale = p.softmax_scale < 0.f ? -p.softmax_scale : p.softmax_scale;
  A.scale_log2 = (abs_scale > 0.f ? abs_scale : 1e-30f) * kLog2e;
  A.negate_s = p.softmax_scale < 0.f ? 1u : 0u;
  A.epi = make_epilogue(p.epilogue, p.n_epilogue);
  A.wd = ctx.wd;
  const long long n_pairs = A.two_tiles ? p.hq / 2 : p.hq;
  const long long items = static_cast<long long>(A.n_qblocks) * p.batch * n_pairs;
  if (items == 0) return FA_OK;
  if (items > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  // persistent: one CTA per SM (the shared memory allows no second), each
  // walking its share of the items
  const long long grid = items < device_sm_count() ? items : device_sm_count();
  auto kern = prefill_tc_kernel<D, kI8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem) != cudaSuccess)
    return FA_ERR_CUDA;
  note_variant(reinterpret_cast<const void*>(kern));
  kern<<<static_cast<unsigned>(grid), G::kThreads, G::kSmem, ctx.stream>>>(tq, tk, tv, A);
  return cuda_status(cudaGetLastError());
}

}  // namespace

fa_status launch_prefill_tc(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink,
                            const LaunchCtx& ctx) {
  if (p.kv_dtype == FA_I8) {
    if (p.head_dim == 128) return launch_tc<128, true>(p, pages, sink, ctx);
    if (p.head_dim == 64) return launch_tc<64, true>(p, pages, sink, ctx);
    return FA_ERR_UNSUPPORTED;
  }
  if (p.head_dim == 128) return launch_tc<128, false>(p, pages, sink, ctx);
  if (p.head_dim == 64) return launch_tc<64, false>(p, pages, sink, ctx);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
