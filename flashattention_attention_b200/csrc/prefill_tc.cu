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
// Above d = 128 two O tiles no longer fit beside their S tiles: one Q tile
// per CTA and 64-key K/V tiles (S [0,64), O [64,64+D)).
//
// Operand tiles are 64-dim chunks in the 128-byte swizzle; a 32-dim remainder
// of the head size is one more such chunk whose upper half the TMA fills
// with zeros (int8 K/V at d = 96: a 32-dim chunk in the 64-byte swizzle).
// L2 policies: Q loads evict_first (read once), K/V loads evict_last (read
// again by later q-blocks and the group's other head pairs), output stores
// evict_first.
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
// dequantise it as c * s in fp32 (dequant4_bf16 below), round it to bf16,
// the tensor-core operand type, write it in the operand layout and fence it
// to the async proxy.  The softmax is then the bf16 one.
// That variant runs 16 warps and rebalances registers with setmaxnreg
// (softmax 176, the rest 80).  Above d = 128 (one Q tile, 64-key tiles, 16
// warps) two converter threads share a key row, and the int8 tiles land in
// rings of their own so the bf16 operand slots fit beside the Q tile.
#include <cstdlib>
#include <mutex>

#include "internal.h"
#include "layout.cuh"
#include "umma.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per Q tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kChunkBytes = kSwizzleChunkRows * 128;  // [128 rows x 64 bf16]

// BN keys per K/V tile, NT Q tiles (query heads) per CTA.  Warps 0 .. 4 NT - 1
// run the softmax (four per Q tile), then the producer, the MMA issuer and,
// for int8 K/V, two idle warps and four converters.
template <int D, bool kI8, bool kPair = false, int BN_ = 128, int NT_ = 2>
struct TcGeom {
  static constexpr int BN = BN_;
  static constexpr int NT = NT_;
  static constexpr int kLoadWarp = 4 * NT;
  static constexpr int kMmaWarp = 4 * NT + 1;
  static constexpr int kConvWarp0 = 4 * NT + 4;
  // K is consumed one step before V (S(j) precedes PV(j)), so K gets the
  // deeper ring: a slot refills with the TMA latency hidden behind ~2 steps.
  // A CTA of a pair holds half of every K and V tile (64 keys of K, 64 dims
  // of V), so its rings can be deeper.
  static constexpr int kKStages = kPair ? (kI8 ? 3 : 4)
                                 : (NT == 4 ? 6 : ((kI8 && D == 96) || D > 128 ? 2 : 3));
  static constexpr int kVStages = kPair ? (kI8 ? 3 : 4)
                                 : (NT == 4 ? 6 : (kI8 && D > 128 ? 1 : ((D == 128 || D == 96 || D > 128) ? 2 : 3)));
  // int8 above d = 128: the int8 tiles land in rings of their own (a slot
  // is refilled once the converters have read it), so the bf16 operand slots
  // (one V slot, two K slots) fit beside a 64 KB Q tile; otherwise an int8
  // tile and its bf16 slot share the ring position
  static constexpr bool kSplitRaw = kI8 && D > 128;
  static constexpr int kRawKStages = !kI8 ? 0 : (kSplitRaw ? 2 : kKStages);
  static constexpr int kRawVStages = !kI8 ? 0 : (kSplitRaw ? 2 : kVStages);
  // D = 64 kNFull + 32 kTail: kNFull chunks of 64 dims (128-byte rows,
  // 128-byte swizzle), then, for an odd multiple of 32, a 32-dim tail: as a
  // further 64-dim chunk whose upper half TMA fills with zeros (one PV MMA
  // with N = D), except with int8 K/V at d = 96, whose separate int8
  // staging leaves no room for padded slots: there the tail is a chunk of
  // 32 dims (64-byte rows, 64-byte swizzle) with MMAs of its own
  static constexpr int kNFull = D / 64;
  static constexpr bool kTail = (D % 64) == 32;
  static constexpr bool kTailSw64 = kTail && kI8 && D == 96;
  static constexpr int kNChunks = kNFull + ((kTail && !kTailSw64) ? 1 : 0);  // 128-byte-swizzled chunks
  static constexpr int kDP = kTailSw64 ? D : 64 * kNChunks;                  // dims per staged bf16 row
  static_assert(D % 32 == 0, "head size");
  static constexpr uint32_t kQBytes = kBM * kDP * 2;
  static constexpr int kKRows = kPair ? BN / 2 : BN;               // K rows in this CTA's slot
  static constexpr uint32_t kKChunk = kKRows * 128;                 // one 64-dim chunk of them
  static constexpr uint32_t kKBytes = kKRows * kDP * 2;             // this CTA's bf16 K slot
  static constexpr uint32_t kVChunk = BN * 128;                     // 64 dims of every key of a tile
  static constexpr uint32_t kVBytes = BN * (kPair ? D / 2 : kDP) * 2;  // this CTA's bf16 V slot
  static constexpr uint32_t kKI8Bytes = kKRows * D;                 // the int8 tiles (unpadded rows)
  static constexpr uint32_t kVI8Bytes = BN * (kPair ? D / 2 : D);
  static constexpr uint32_t kKOff = NT * kQBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kKBytes;
  // int8 staging: at d = 128 (one CTA) in the upper half of each bf16 slot
  // (a row's bf16 output overwrites only that row's int8 bytes); otherwise
  // separate
  static constexpr bool kInPlace = (D == 128) && !kPair;
  static constexpr uint32_t kStageOff = kVOff + kVStages * kVBytes;
  static constexpr uint32_t kStageBytes =
      (kI8 && !kInPlace) ? kRawKStages * kKI8Bytes + kRawVStages * kVI8Bytes : 0;
  static constexpr uint32_t kBarOff = kStageOff + kStageBytes;
  // mbarriers (8 bytes each, the order of the kernel's pointers) + the TMEM address
  static constexpr uint32_t kBarBytes =
      8 * (1 + 2 * kKStages + 2 * kVStages + 5 * NT + 1 + 2 * kRawKStages + 2 * kRawVStages + 1) + 4;
  static_assert(kBarBytes <= 512, "barrier area");
  static constexpr uint32_t kSmem = kBarOff + 512 + 1024;
  // int8: 2 idle warps and 4 converters; four Q tiles: a fifth warpgroup
  // (producer, MMA, 2 idle) so registers can move between warpgroups
  // (int8 above 128: 2 idle warps, 4 K converters and 4 V converters)
  static constexpr int kThreads = (4 * NT + ((kI8 || NT == 4) ? (kI8 ? (kSplitRaw ? 12 : 8) : 4) : 2)) * 32;
  // setmaxnreg split (0: none): the softmax warpgroups take kRegsHi, the
  // others give back down to 64 (the totals match the launch's pool)
  // (int8, two Q tiles: 2 x 128 threads at 176, 2 x 128 at 80 = 512 * 128;
  // with one Q tile, 512 threads: one softmax warpgroup at 192, three at 96)
  static constexpr int kRegsHi = kI8 ? (kSplitRaw ? 192 : 176) : (NT == 4 ? 104 : 0);
  static constexpr int kRegsLo = kSplitRaw ? 96 : (NT == 4 ? 64 : 80);
  // the registers a launch of kThreads threads gets per thread, which the
  // split redistributes (setmaxnreg.inc waits for registers the pool lacks)
  static constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
  static_assert(kRegsHi == 0 || 128 * NT * kRegsHi + (kThreads - 128 * NT) * kRegsLo <= kThreads * kLaunchRegs,
                "setmaxnreg budget");
  // TMEM columns: S_t (P_t over its first BN / 2 columns) and O_t
  static constexpr uint32_t s_col(int t) { return t * BN; }
  static constexpr uint32_t o_col(int t) { return NT * BN + t * D; }
  static_assert(NT * (BN + D) <= 512, "TMEM columns");
  __host__ __device__ static constexpr uint32_t k_stage(int s) {
    return kInPlace ? kKOff + s * kKBytes + kKBytes / 2 : kStageOff + s * kKI8Bytes;
  }
  __host__ __device__ static constexpr uint32_t v_stage(int s) {
    return kInPlace ? kVOff + s * kVBytes + kVBytes / 2 : kStageOff + kRawKStages * kKI8Bytes + s * kVI8Bytes;
  }
};
static_assert(TcGeom<128, false>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<128, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<64, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<128, false, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<128, true, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<64, false, false, 64, 4>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<96, false>::kSmem <= 232448 && TcGeom<96, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<32, true>::kSmem <= 232448, "shared memory budget");
static_assert(TcGeom<256, false, false, 64, 1>::kSmem <= 232448 && TcGeom<224, false, false, 64, 1>::kSmem <= 232448,
              "shared memory budget");
static_assert(TcGeom<256, true, false, 64, 1>::kSmem <= 232448 && TcGeom<224, true, false, 64, 1>::kSmem <= 232448,
              "shared memory budget");
static_assert(TcGeom<160, false, false, 64, 1>::kSmem <= 232448 && TcGeom<160, true, false, 64, 1>::kSmem <= 232448 &&
                  TcGeom<192, true, false, 64, 1>::kSmem <= 232448 && TcGeom<32, false>::kSmem <= 232448,
              "shared memory budget");

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
  int heads_per_item;    // 1, 2 (head pair), or 4 (CTA pair: two heads per CTA)
  float scale_log2;      // |softmax scale| * log2(e), > 0
  uint32_t negate_s;     // 1: the MMA negates Q (a negative softmax scale)
  Epilogue epi;
  Watchdog wd;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Four signed bytes of w times the row scale, as bf16 (two bf16x2 words).
// Each byte b, flipped to b ^ 0x80 = c + 128, is placed in the low mantissa
// byte of 2^23, so the float is 2^23 + 128 + c and one exact subtraction
// leaves c.  c * s is rounded to fp32 (a 7-bit |c| times a 24-bit
// significand can need 31 bits) and then to bf16; that differs from one
// rounding of c * s to bf16 only when the fp32 result lands exactly halfway
// between two bf16 values, by one bf16 unit in the last place.
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

// NC 16-byte chunks of int8 codes, from chunk c0 of row `row` of a staged
// tile with RL-byte rows (128- or 64-byte swizzle as TMA wrote it), times the
// row's scale, rounded to bf16 and written as pieces of output chunk c / 4
// (128-byte rows with the 128-byte swizzle, chunks dst_chunk bytes apart).
// Each thread reads its own row's bytes before writing that row.
template <int NC, int RL, int kNFull = 8>
__device__ __forceinline__ void convert_int8_row(const uint8_t* src_tile, uint8_t* dst_tile, uint32_t dst_chunk,
                                                 int row, int c0, float sc) {
  const float2 s2 = make_float2(sc, sc);
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = c0 + i;
    // staged row: 128-, 64- or 32-byte swizzle (RL = 128, 64, 32), plain rows otherwise
    const int pc = (RL == 128) ? (c ^ (row & 7))
                 : (RL == 64) ? (c ^ ((row >> 1) & 3))
                 : (RL == 32) ? (c ^ ((row >> 2) & 1))
                              : c;
    const uint4 w = *reinterpret_cast<const uint4*>(src_tile + row * RL + pc * 16);
    const int h = c / 4, j0 = 2 * (c % 4);
    const uint2 y0 = dequant4_bf16(w.x, s2), y1 = dequant4_bf16(w.y, s2);
    const uint2 y2 = dequant4_bf16(w.z, s2), y3 = dequant4_bf16(w.w, s2);
    if (h < kNFull) {  // a 64-dim chunk: 128-byte rows, 128-byte swizzle
      uint8_t* out = dst_tile + h * dst_chunk + row * 128;
      *reinterpret_cast<uint4*>(out + ((j0 ^ (row & 7)) * 16)) = make_uint4(y0.x, y0.y, y1.x, y1.y);
      *reinterpret_cast<uint4*>(out + (((j0 + 1) ^ (row & 7)) * 16)) = make_uint4(y2.x, y2.y, y3.x, y3.y);
    } else {  // the 32-dim tail: 64-byte rows, 64-byte swizzle
      uint8_t* out = dst_tile + h * dst_chunk + row * 64;
      const int sw = (row >> 1) & 3;
      *reinterpret_cast<uint4*>(out + ((j0 ^ sw) * 16)) = make_uint4(y0.x, y0.y, y1.x, y1.y);
      *reinterpret_cast<uint4*>(out + (((j0 + 1) ^ sw) * 16)) = make_uint4(y2.x, y2.y, y3.x, y3.y);
    }
  }
}

// Above d = 128 (64-key tiles, int8 rows staged without swizzle, D bytes
// each): thread (row, h) converts D / 32 of the row's D / 16 chunks of 16
// codes, chunk c0 + 2i (mod D / 16) at step i, with c0 = h + a row + b h +
// f (row / 2).  The two threads of a row cover it once; a, b, f were found
// by an exhaustive search so that the 8 lanes of each shared-memory phase
// (4 rows x 2 halves) read 8 different bank groups, and write at most 2 to
// one (2 only at d = 160 and 224; no order of this family does better).
template <int D, int kNFull>
__device__ __forceinline__ void convert_int8_half_row(const uint8_t* src_tile, uint8_t* dst_tile, uint32_t dst_chunk,
                                                      int row, int h, float sc) {
  constexpr int U = D / 16;
  constexpr int a = D == 256 ? 2 : 0, b = D == 256 ? 2 : 0, f = D == 192 ? 2 : 0;
  const float2 s2 = make_float2(sc, sc);
  const uint8_t* src = src_tile + row * D;
  int c = (h + a * row + b * h + f * (row >> 1)) % U;
#pragma unroll
  for (int i = 0; i < U / 2; ++i) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + c * 16);
    const uint2 y0 = dequant4_bf16(w.x, s2), y1 = dequant4_bf16(w.y, s2);
    const uint2 y2 = dequant4_bf16(w.z, s2), y3 = dequant4_bf16(w.w, s2);
    const int hc = c >> 2, j0 = 2 * (c & 3);
    // a 64-dim chunk: 128-byte rows, 128-byte swizzle; the 32-dim tail:
    // 64-byte rows, 64-byte swizzle
    const bool tail = hc >= kNFull;
    const int sw = tail ? ((row >> 1) & 3) : (row & 7);
    uint8_t* out = dst_tile + hc * dst_chunk + row * (tail ? 64 : 128);
    *reinterpret_cast<uint4*>(out + ((j0 ^ sw) * 16)) = make_uint4(y0.x, y0.y, y1.x, y1.y);
    *reinterpret_cast<uint4*>(out + (((j0 + 1) ^ sw) * 16)) = make_uint4(y2.x, y2.y, y3.x, y3.y);
    c += 2;
    if (c >= U) c -= U;
  }
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
// In a CTA pair, CTA `rank` takes heads 2 rank and 2 rank + 1 of the item's
// four (all of one GQA group: the group size is a multiple of 4).
template <int BN>
__device__ __forceinline__ bool item_of(const PrefillArgs& A, int item, Item& w, int rank = 0) {
  const int n_sets = A.hq / A.heads_per_item;
  const int per_qb = A.batch * n_sets;
  const int qb = A.n_qblocks - 1 - item / per_qb;
  const int rem = item % per_qb;
  w.b = rem / n_sets;
  const int set = rem % n_sets;
  w.h0 = A.heads_per_item * set + 2 * rank;
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
  w.j_lo = k_lo / BN;
  w.n_iter = k_hi > k_lo ? (k_hi + BN - 1) / BN - w.j_lo : 0;
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

// TMA plane and row of the key tile starting at key0 of item w (paged:
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

template <int D, bool kI8, bool kPair, int BN, int NT>
__global__ void __launch_bounds__(TcGeom<D, kI8, kPair, BN, NT>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q32,
                      const PrefillArgs A) {
  using G = TcGeom<D, kI8, kPair, BN, NT>;
  constexpr int KS = G::kKStages, VS = G::kVStages, RKS = G::kRawKStages, RVS = G::kRawVStages;
  constexpr int kLoadWarp = G::kLoadWarp, kMmaWarp = G::kMmaWarp, kConvWarp0 = G::kConvWarp0;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;  // [NT]
  uint64_t* p_full = s_full + NT;  // [NT tiles][2 halves of the keys]
  uint64_t* o_done = p_full + 2 * NT;  // [NT]
  uint64_t* drain = o_done + NT;
  uint64_t* kraw_full = drain + 1;   // [RKS] int8 variant: TMA landed the int8 K tile
  uint64_t* vraw_full = kraw_full + RKS;
  uint64_t* kraw_empty = vraw_full + RVS;  // [RKS] separate int8 rings: the converters have read it
  uint64_t* vraw_empty = kraw_empty + RKS;
  uint64_t* q_empty = vraw_empty + RVS;  // every S MMA of an item has read Q
  uint64_t* o_free = q_empty + 1;       // [NT] the softmax warps have read O_t out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_free + NT);
  __shared__ int abort_flag;

  // A CTA pair (cluster of two) runs M = 256 MMAs: CTA 0 issues them and owns
  // the barriers they wait on; CTA 1's producer, converters and softmax warps
  // signal those barriers remotely, and every MMA completion is signalled to
  // the same barrier in both CTAs.
  const int rank = kPair ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = rank == 0;
  auto lead = [&](uint64_t* b) -> uint32_t { return kPair ? mapa_shared(smem_u32(b), 0) : smem_u32(b); };
  // a barrier of the issuing CTA that some arrivals reach from the peer CTA
  auto wait_x = [&](uint64_t* b, uint32_t ph) -> bool {
    return kPair ? wait_parity<true>(b, ph, A.wd, &abort_flag) : wait_parity(b, ph, A.wd, &abort_flag);
  };
  // warp-level arrival on a barrier counted per thread (one CTA) or per warp
  // of both CTAs (pair); the caller has made its TMEM / smem writes visible
  auto arrive_x = [&](uint64_t* b) {
    if constexpr (kPair) {
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(lead(b));
    } else {
      mbar_arrive(b);
    }
  };
  auto commit = [&](uint64_t* b) {
    if constexpr (kPair) mma_commit_pair_both(b);
    else mma_commit(b);
  };
  // Persistent CTAs (pairs): unit u takes one item per round of n_units items
  // of the longest-first order (item_at); every role of both CTAs of a pair
  // walks the same sequence, with the K/V ring and every barrier phase
  // counted across items.
  const int unit = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int n_units = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int n_items = A.n_qblocks * A.batch * (A.hq / A.heads_per_item);
  const int ntile = kPair ? 2 : A.heads_per_item;
  constexpr uint32_t kArrivals = kPair ? 8 : kBM;  // warps of both CTAs, or threads of one

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    // bf16: TMA completes k_full / v_full; int8: the converter threads do
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, kI8 ? kArrivals : 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, kI8 ? kArrivals : 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < RKS; ++s) {
      mbar_init(kraw_full + s, 1);
      mbar_init(kraw_empty + s, kArrivals);
    }
    for (int s = 0; s < RVS; ++s) {
      mbar_init(vraw_full + s, 1);
      mbar_init(vraw_empty + s, kArrivals);
    }
    for (int t = 0; t < NT; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + 2 * t, kArrivals);
      mbar_init(p_full + 2 * t + 1, kArrivals);
      mbar_init(o_done + t, 1);
      mbar_init(o_free + t, kArrivals);
    }
    mbar_init(drain, 1);
    mbar_init(q_empty, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    if constexpr (kPair) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Roles split by warpgroup first: the first NT warpgroups softmax, the rest
  // the other roles, which give registers back to the softmax warpgroups
  // where TcGeom sets a split (kRegsHi / kRegsLo).
  if (warp >= 4 * NT) {
  if constexpr (G::kRegsHi > 0) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(G::kRegsLo) : "memory");
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      // every K/V tile is read again by the later q-blocks of its sequence
      // (and the other head pairs of its group), each Q tile once: K/V stay
      // in L2 ahead of the Q stream
      const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
      int base = 0, done = 0;  // K/V tiles and items before this one
      bool ok = true;
      for (int k = 0, item; ok && (item = item_at(unit, n_units, k)) < n_items; ++k) {
        Item w;
        if (!item_of<BN>(A, item, w, rank)) continue;
        // Q of this item once every S MMA of the previous one has read its Q
        if (done > 0 && !wait_parity<kPair>(q_empty, (done - 1) & 1, A.wd, &abort_flag)) break;
        if (leader) mbar_expect_tx(q_full, (kPair ? 2 : 1) * ntile * G::kQBytes);
        for (int t = 0; t < ntile; ++t) {
          for (int c = 0; c < G::kNChunks; ++c) {
            uint8_t* dst = smem + t * G::kQBytes + c * kChunkBytes;
            if constexpr (kPair) tma_load_3d_pair(dst, &tm_q, lead(q_full), 64 * c, w.q_prow, w.q_plane + t);
            else tma_load_3d_hint(dst, &tm_q, q_full, 64 * c, w.q_prow, w.q_plane + t, pol_q);
          }
          if constexpr (G::kTailSw64)
            tma_load_3d_hint(smem + t * G::kQBytes + G::kNFull * kChunkBytes, &tm_q32, q_full, 64 * G::kNFull,
                             w.q_prow, w.q_plane + t, pol_q);
        }
        for (int it = 0; it < w.n_iter; ++it) {
          const int gi = base + it;
          int s = gi % KS, u = gi / KS;
          int kplane, krow;
          kv_tile(A, w, (w.j_lo + it) * BN, kplane, krow);
          if constexpr (G::kSplitRaw) {
            // separate int8 ring: its slot is free once the converters read it
            s = gi % RKS;
            u = gi / RKS;
            if (u > 0 && !(ok = wait_parity(kraw_empty + s, (u - 1) & 1, A.wd, &abort_flag))) break;
          } else if (u > 0 && !(ok = wait_parity<kPair>(k_empty + s, (u - 1) & 1, A.wd, &abort_flag))) {
            break;
          }
          // a pair's CTA r brings keys [64 r, 64 r + 64) of K and dims
          // [D/2 r, D/2 r + D/2) of V
          const int k_row = krow + (kPair ? 64 * rank : 0);
          if constexpr (kI8) {
            mbar_expect_tx(kraw_full + s, G::kKI8Bytes);
            tma_load_3d_hint(smem + G::k_stage(s), &tm_k, kraw_full + s, 0, k_row, kplane, pol_kv);
          } else if constexpr (kPair) {
            if (leader) mbar_expect_tx(k_full + s, 2 * G::kKBytes);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d_pair(smem + G::kKOff + s * G::kKBytes + c * G::kKChunk, &tm_k, lead(k_full + s), 64 * c,
                               k_row, kplane);
          } else {
            mbar_expect_tx(k_full + s, G::kKBytes);
            // (a padded tail chunk: the dims past D read as zeros)
            for (int c = 0; c < G::kNChunks; ++c)
              tma_load_3d_hint(smem + G::kKOff + s * G::kKBytes + c * G::kKChunk, &tm_k, k_full + s, 64 * c, krow,
                               kplane, pol_kv);
          }
          if constexpr (G::kSplitRaw) {
            s = gi % RVS;
            u = gi / RVS;
            if (u > 0 && !(ok = wait_parity(vraw_empty + s, (u - 1) & 1, A.wd, &abort_flag))) break;
          } else {
            s = gi % VS;
            u = gi / VS;
            if (u > 0 && !(ok = wait_parity<kPair>(v_empty + s, (u - 1) & 1, A.wd, &abort_flag))) break;
          }
          if constexpr (kI8) {
            mbar_expect_tx(vraw_full + s, G::kVI8Bytes);
            tma_load_3d_hint(smem + G::v_stage(s), &tm_v, vraw_full + s, kPair ? (D / 2) * rank : 0, krow, kplane,
                             pol_kv);
          } else if constexpr (kPair) {
            if (leader) mbar_expect_tx(v_full + s, 2 * G::kVBytes);
            tma_load_3d_pair(smem + G::kVOff + s * G::kVBytes, &tm_v, lead(v_full + s), (D / 2) * rank, krow, kplane);
          } else {
            mbar_expect_tx(v_full + s, G::kVBytes);
            for (int c = 0; c < G::kNChunks; ++c)
              tma_load_3d_hint(smem + G::kVOff + s * G::kVBytes + c * G::kVChunk, &tm_v, v_full + s, 64 * c, krow,
                               kplane, pol_kv);
          }
        }
        base += w.n_iter;
        ++done;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      // a negative softmax scale is folded into the S MMA (negated A operand),
      // so the softmax only ever sees a positive scale
      constexpr int kM = kPair ? 2 * kBM : kBM;
      const uint32_t idesc_s = umma_idesc_f16(kM, BN, 1, 1, false) | (A.negate_s << 13);
      // PV: one MMA over every dim (N = D; a padded tail chunk's upper half
      // is never read), or, with a 64-byte-swizzled tail, the 64-dim chunks
      // (N = 64 kNFull) and the tail (N = 32)
      constexpr uint32_t idesc_o =
          umma_idesc_f16(kM, G::kTailSw64 ? (G::kNFull > 0 ? 64 * G::kNFull : 32) : D, 1, 1, true);
      // S: 16-dim k-steps over the 128-byte-swizzled chunks (2 in a padded tail)
      constexpr int kSSteps = 4 * G::kNFull + ((G::kTail && !G::kTailSw64) ? 2 : 0);
      constexpr uint32_t idesc_o32 = umma_idesc_f16(kM, 32, 1, 1, true);
      const uint32_t q_base = smem_u32(smem);
      // operand descriptors are built once; a k-step only moves the start
      // address (its 14-bit field never carries: every address is < 2^18)
      const uint64_t dq0 = umma_desc_sw128(q_base, 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(q_base + G::kKOff, 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(q_base + G::kVOff, G::kVChunk, 1024);
      // 64-byte-swizzled 32-dim tails (int8 K/V at d = 96): Q of tile 0, K and V of stage 0
      const uint64_t dq32 = umma_desc_sw64(q_base + G::kNFull * kChunkBytes, 16, 512);
      const uint64_t dk32 = umma_desc_sw64(q_base + G::kKOff + G::kNFull * G::kKChunk, 16, 512);
      const uint64_t dv32 = umma_desc_sw64(q_base + G::kVOff + G::kNFull * G::kVChunk, 16, 512);
      auto issue_s = [&](int t, int st) {
        const uint64_t dq = dq0 + ((t * G::kQBytes) >> 4);
        const uint64_t dk = dk0 + ((st * G::kKBytes) >> 4);
#pragma unroll
        for (int k = 0; k < kSSteps; ++k) {
          const uint32_t off_q = ((k / 4) * kChunkBytes + (k % 4) * 32) >> 4;
          const uint32_t off_k = ((k / 4) * G::kKChunk + (k % 4) * 32) >> 4;
          if constexpr (kPair) mma_ss_pair(tmem + G::s_col(t), dq + off_q, dk + off_k, idesc_s, k > 0 ? 1u : 0u);
          else mma_ss(tmem + G::s_col(t), dq + off_q, dk + off_k, idesc_s, k > 0 ? 1u : 0u);
        }
        if constexpr (G::kTailSw64) {
          const uint64_t tq = dq32 + ((t * G::kQBytes) >> 4), tk = dk32 + ((st * G::kKBytes) >> 4);
#pragma unroll
          for (int k = 0; k < 2; ++k)
            mma_ss(tmem + G::s_col(t), tq + ((k * 32) >> 4), tk + ((k * 32) >> 4), idesc_s,
                   (G::kNFull > 0 || k > 0) ? 1u : 0u);
        }
      };
      // O_t += P_t V over keys [BN/2 h, BN/2 h + BN/2) (16-key MMA steps)
      auto issue_pv_half = [&](int t, int st, int h, bool accumulate) {
        const uint64_t dv = dv0 + ((st * G::kVBytes) >> 4);
        constexpr int kHalf = BN / 32;
#pragma unroll
        for (int k = kHalf * h; k < kHalf * h + kHalf; ++k) {
          const uint32_t acc = (accumulate || k > 0) ? 1u : 0u;
          if constexpr (kPair) {
            mma_ts_pair(tmem + G::o_col(t), tmem + G::s_col(t) + k * 8, dv + ((k * 2048) >> 4), idesc_o, acc);
          } else {
            if constexpr (G::kNChunks > 0)
              mma_ts(tmem + G::o_col(t), tmem + G::s_col(t) + k * 8, dv + ((k * 2048) >> 4), idesc_o, acc);
            if constexpr (G::kTailSw64)
              mma_ts(tmem + G::o_col(t) + 64 * G::kNFull, tmem + G::s_col(t) + k * 8,
                     dv32 + ((st * G::kVBytes + k * 1024) >> 4), idesc_o32, acc);
          }
        }
      };
      int base = 0, done = 0;  // K/V tiles and items before the current one
      // PV for step j (of the current item) of tile t, each half as soon as
      // the softmax wrote it; an item's first PV overwrites O_t, so it also
      // waits until the previous item's O_t has been read out
      auto issue_pv = [&](int t, int j) -> bool {
        const int gj = base + j;
        const int vs = gj % VS;
        if (j == 0 && done > 0 && !wait_x(o_free + t, (done - 1) & 1)) return false;
        if (!wait_x(p_full + 2 * t, gj & 1)) return false;
        if (t == 0 && !wait_x(v_full + vs, (gj / VS) & 1)) return false;
        tc_fence_after();
        issue_pv_half(t, vs, 0, j > 0);
        if (!wait_x(p_full + 2 * t + 1, gj & 1)) return false;
        tc_fence_after();
        issue_pv_half(t, vs, 1, true);
        return true;
      };
      bool ok = true;
      for (int k = 0, item; ok && (item = item_at(unit, n_units, k)) < n_items; ++k) {
        Item w;
        if (!item_of<BN>(A, item, w, rank)) continue;
        if (!(ok = wait_x(q_full, done & 1))) break;
        for (int it = 0; ok && it < w.n_iter; ++it) {
          const int gi = base + it;
          const int s = gi % KS;
          if (!(ok = wait_x(k_full + s, (gi / KS) & 1))) break;
          tc_fence_after();
          for (int t = 0; t < ntile; ++t) {
            if (it > 0) {
              if (!(ok = issue_pv(t, it - 1))) break;
              if (t == ntile - 1) commit(v_empty + (gi - 1) % VS);
            }
            issue_s(t, s);
            commit(s_full + t);
          }
          if (ok) commit(k_empty + s);
        }
        if (!ok) break;
        commit(q_empty);  // Q is free once this item's S MMAs complete
        for (int t = 0; t < ntile; ++t) {
          if (!(ok = issue_pv(t, w.n_iter - 1))) break;
          commit(o_done + t);
        }
        if (!ok) break;
        commit(v_empty + (base + w.n_iter - 1) % VS);
        base += w.n_iter;
        ++done;
      }
      // every MMA this thread issued has completed before TMEM is released
      commit(drain);
      wait_parity(drain, 0, A.wd);
    }
  } else if (G::kSplitRaw && warp >= kConvWarp0) {
    // ------------------------------------------------------------ int8 -> bf16 converters, d > 128
    // Warps kConvWarp0 .. +3 convert K, the next four V, two threads per
    // key row of the 64-key tiles.  A tile's int8 slot is released once
    // read; its bf16 slot is written once the MMAs that read the slot's
    // previous tile have completed.
    const int r = static_cast<int>(threadIdx.x) - kConvWarp0 * 32;
    const bool is_v = r >= 128;  // warp-uniform
    const int row = (r & 127) >> 1, h = r & 1;
    uint64_t* raw_full = is_v ? vraw_full : kraw_full;
    uint64_t* raw_empty = is_v ? vraw_empty : kraw_empty;
    uint64_t* op_full = is_v ? v_full : k_full;
    uint64_t* op_empty = is_v ? v_empty : k_empty;
    const int n_raw = is_v ? RVS : RKS, n_op = is_v ? VS : KS;
    const float* scales = is_v ? A.v_scales : A.k_scales;
    static_assert(!G::kSplitRaw ||
                      (G::kKChunk == G::kVChunk && G::kKBytes == G::kVBytes && G::kKI8Bytes == G::kVI8Bytes),
                  "K and V slots alike");
    const uint32_t op_off = is_v ? G::kVOff : G::kKOff;
    int base = 0;
    bool ok = true;
    for (int k = 0, item; ok && (item = item_at(unit, n_units, k)) < n_items; ++k) {
      Item w;
      if (!item_of<BN>(A, item, w, rank)) continue;
      for (int it = 0; it < w.n_iter; ++it) {
        const int gi = base + it;
        const int key0 = (w.j_lo + it) * BN;
        float sc = 0.f;  // 0 past the sequence end: those rows become zeros
        if (key0 + row < w.sq.s_k) {
          int kplane, krow;
          kv_tile(A, w, key0, kplane, krow);
          sc = __ldg(scales + static_cast<int64_t>(kplane) * A.k_plane_rows + krow + row);
        }
        const int rs = gi % n_raw, s = gi % n_op;
        if (!(ok = __all_sync(0xffffffffu, wait_parity(raw_full + rs, (gi / n_raw) & 1, A.wd, &abort_flag)))) break;
        if (gi >= n_op &&
            !(ok = __all_sync(0xffffffffu, wait_parity(op_empty + s, (gi / n_op - 1) & 1, A.wd, &abort_flag))))
          break;
        convert_int8_half_row<D, G::kNChunks>(smem + (is_v ? G::v_stage(rs) : G::k_stage(rs)),
                                            smem + op_off + s * G::kKBytes, G::kKChunk, row, h, sc);
        fence_proxy_async_smem();
        mbar_arrive(raw_empty + rs);
        mbar_arrive(op_full + s);
      }
      base += w.n_iter;
    }
  } else if (kI8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ int8 -> bf16 converters
    // One CTA: thread r rewrites key row r of each int8 K and V tile as bf16
    // in the 128-byte-swizzled K-major (K) / MN-major (V) operand layout.
    // Pair: this CTA's K slot holds 64 key rows (thread r converts half row
    // r / 2, dims [64 (r % 2), +64)) and its V slot 64 dims of 128 key rows
    // (thread r converts row r).
    const int r = static_cast<int>(threadIdx.x) - kConvWarp0 * 32;
    const int k_r = kPair ? r / 2 : r;                  // K row this thread converts
    const int k_c0 = kPair ? (r % 2) * 4 : 0;           // its first 16-byte chunk
    constexpr int k_nc = kPair ? 4 : D / 16;
    constexpr int v_rl = kPair ? D / 2 : D;             // staged V row bytes
    int base = 0;
    bool ok = true;
    for (int k = 0, item; ok && (item = item_at(unit, n_units, k)) < n_items; ++k) {
      Item w;
      if (!item_of<BN>(A, item, w, rank)) continue;
      for (int it = 0; it < w.n_iter; ++it) {
        const int gi = base + it;
        const int s = gi % KS, sv = gi % VS;
        const uint32_t ph = (gi / KS) & 1, phv = (gi / VS) & 1;
        // this thread's key rows: their scales, loaded ahead of the waits (0
        // past the sequence end, so those rows become zeros; the softmax masks them)
        const int key0 = (w.j_lo + it) * BN;
        const int kkey = key0 + (kPair ? 64 * rank : 0) + k_r, vkey = key0 + r;
        float ksc = 0.f, vsc = 0.f;
        {
          int kplane, krow;
          kv_tile(A, w, key0, kplane, krow);
          const int64_t at = static_cast<int64_t>(kplane) * A.k_plane_rows + krow;
          if (kkey < w.sq.s_k) ksc = __ldg(A.k_scales + at + (kkey - key0));
          if (vkey < w.sq.s_k) vsc = __ldg(A.v_scales + at + r);
        }
        if (!(ok = __all_sync(0xffffffffu, wait_parity(kraw_full + s, ph, A.wd, &abort_flag)))) break;
        convert_int8_row<k_nc, D, G::kNChunks>(smem + G::k_stage(s), smem + G::kKOff + s * G::kKBytes, G::kKChunk,
                                             k_r, k_c0, ksc);
        fence_proxy_async_smem();
        arrive_x(k_full + s);
        if (!(ok = __all_sync(0xffffffffu, wait_parity(vraw_full + sv, phv, A.wd, &abort_flag)))) break;
        convert_int8_row<v_rl / 16, v_rl, kPair ? 8 : G::kNChunks>(smem + G::v_stage(sv),
                                                                 smem + G::kVOff + sv * G::kVBytes, G::kVChunk, r, 0,
                                                                 vsc);
        fence_proxy_async_smem();
        arrive_x(v_full + sv);
      }
      base += w.n_iter;
    }
  }
  } else {
  if constexpr (G::kRegsHi > 0) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(G::kRegsHi) : "memory");
  if (warp / 4 < ntile) {
    // ------------------------------------------------------------ softmax
    const int t = warp / 4, quarter = warp % 4;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + G::s_col(t);
    const uint32_t o_tm = tmem + lane_base + G::o_col(t);
    int base = 0, done = 0;  // K/V tiles and items before the current one
    bool ok = true;
    for (int k = 0, item; ok && (item = item_at(unit, n_units, k)) < n_items; ++k) {
    Item w;
    if (!item_of<BN>(A, item, w, rank)) continue;
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
      ok = __all_sync(0xffffffffu, wait_parity<kPair>(s_full + t, (base + it) & 1, A.wd, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      constexpr int kCh = BN / 32;  // 32-column chunks of the S row
      uint32_t raw[kCh][32];
#pragma unroll
      for (int c = 0; c < kCh; ++c) tmem_ld32(s_tm + 32 * c, raw[c]);
      tmem_wait_ld();
      const int kb = (w.j_lo + it) * BN;
      if (!(kb >= lo && kb + BN <= hi)) {
        // boundary tile: keys outside this row's band become -inf (the
        // softmax scale is positive, so masking before it is the same)
        const int va = lo - kb, vb = hi - kb;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c < va || c >= vb) raw[c / 32][c % 32] = 0xff800000u;
      }
      // row max of the raw scores: BN / 16 independent chains of 3-input max
      float g8[2 * kCh];
#pragma unroll
      for (int k = 0; k < 2 * kCh; ++k) {
        const uint32_t* v = &raw[k / 2][(k % 2) * 16];
        float g = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int e = 3; e < 15; e += 2) g = max3f(g, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        g8[k] = fmaxf(g, __uint_as_float(v[15]));
      }
      float m_raw;
      if constexpr (kCh == 4) {
        m_raw = fmaxf(max3f(g8[0], g8[1], g8[2]), max3f(max3f(g8[3], g8[4], g8[5]), g8[6], g8[7]));
      } else {
        m_raw = fmaxf(max3f(g8[0], g8[1], g8[2]), g8[3]);
      }
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
      constexpr int kL = kCh == 4 ? 8 : 4;  // independent row-sum chains
      float2 lacc[kL];
#pragma unroll
      for (int k = 0; k < kL; ++k) lacc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < kCh; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // p = 2^(s * scale * log2(e) - m): one packed FMA for two scores
          const float2 x = fma2(make_float2(__uint_as_float(raw[cc][2 * e]), __uint_as_float(raw[cc][2 * e + 1])),
                                sc2, nm2);
          const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          lacc[e % kL] = add2(lacc[e % kL], pp);
          pk[e] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st16(s_tm + cc * 16, pk);
        if (cc == kCh / 2 - 1 && it > 0 && __any_sync(0xffffffffu, need)) {
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
        if (cc % (kCh / 2) == kCh / 2 - 1) {
          // keys [BN/2 h, BN/2 h + BN/2) of P are in TMEM: let the PV MMA start on them
          tmem_wait_st();
          tc_fence_before();
          arrive_x(p_full + 2 * t + cc / (kCh / 2));
        }
      }
      if constexpr (kL == 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) lacc[k] = add2(lacc[k], lacc[k + 4]);
      }
      lacc[0] = add2(lacc[0], lacc[2]);
      lacc[1] = add2(lacc[1], lacc[3]);
      lacc[0] = add2(lacc[0], lacc[1]);
      l = l * alpha + (lacc[0].x + lacc[0].y);
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_parity<kPair>(o_done + t, done & 1, A.wd, &abort_flag));
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
        arrive_x(o_free + t);
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
        // written once and never read here: marked to leave L2 before the
        // K/V tiles that later q-blocks read again
        uint4* dst = reinterpret_cast<uint4*>(orow + oc * 32);
        const uint64_t pol_o = l2_policy_evict_first();
#pragma unroll
        for (int v = 0; v < 4; ++v)
          stg_v4_hint(dst + v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]), pol_o);
      }
    }
    base += w.n_iter;
    ++done;
    }
  }
  }

  tc_fence_before();
  __syncthreads();
  // pair: CTA 0's MMAs (all complete: its issuer drained them) wrote this
  // CTA's TMEM and read its shared memory, and this CTA's arrivals reached
  // CTA 0's barriers; neither CTA releases TMEM or exits before both are here
  if constexpr (kPair) cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}



// Clusters of two of this kernel that fit on the device at once (cached per
// device and variant); 0 when the query fails.
template <typename K>
int max_pair_clusters(K kern, uint32_t smem, int threads) {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (cached[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count()));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int D, bool kI8, bool kPair, int BN = 128, int NT = 2>
fa_status launch_tc(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink, const LaunchCtx& ctx) {
  using G = TcGeom<D, kI8, kPair, BN, NT>;
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
  // K boxes: G::kKRows key rows (a pair's CTA takes 64 of each 128-key
  // tile); V boxes: BN keys of 64 dims (one CTA: every dim chunk in turn;
  // pair: this CTA's half)
  const uint32_t krows = static_cast<uint32_t>(G::kKRows);
  if constexpr (kI8) {
    // int8 rows: K boxes of whole rows (D bytes), V boxes of this CTA's
    // dims (D bytes, or D / 2 in a pair): the 128-, 64- or 32-byte swizzle
    // of that width, unswizzled rows otherwise (d = 96 and above 128)
    const uint64_t dims[3] = {static_cast<uint64_t>(D), k_rows, k_planes};
    const uint64_t strides[2] = {static_cast<uint64_t>(D), k_rows * D};
    const uint32_t kbox[3] = {static_cast<uint32_t>(D), krows, 1};
    const uint32_t vw = kPair ? D / 2 : D;
    const uint32_t vbox[3] = {vw, static_cast<uint32_t>(BN), 1};
    auto sw_of = [](uint32_t bytes) {
      return bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
           : bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
           : bytes == 32  ? CU_TENSOR_MAP_SWIZZLE_32B
                          : CU_TENSOR_MAP_SWIZZLE_NONE;
    };
    const CUtensorMapSwizzle ksw = sw_of(D), vsw = sw_of(vw);
    fa_status st = encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p.k, dims, strides, kbox, ksw);
    if (st != FA_OK) return st;
    st = encode_tensor_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p.v, dims, strides, vbox, vsw);
    if (st != FA_OK) return st;
  } else {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), k_rows, k_planes};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, k_rows * D * 2};
    const uint32_t kbox[3] = {64, krows, 1};
    const uint32_t vbox[3] = {64, static_cast<uint32_t>(BN), 1};
    fa_status st = encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.k, dims, strides, kbox,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
    st = encode_tensor_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.v, dims, strides, vbox,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }
  // the 64-byte-swizzled Q tail (int8 K/V at d = 96): boxes of 32 dims, the
  // same rows.  Every other tail is a 64-dim box of tq / tk / tv whose dims
  // past D read as zeros.
  CUtensorMap tq32 = tq;
  if constexpr (G::kTailSw64) {
    const uint64_t qdims[3] = {static_cast<uint64_t>(D), q_rows, q_planes};
    const uint64_t qstr[2] = {static_cast<uint64_t>(D) * 2, q_rows * D * 2};
    const uint32_t qbox[3] = {32, static_cast<uint32_t>(kSwizzleChunkRows), 1};
    fa_status st = encode_tensor_map(&tq32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.q, qdims, qstr, qbox,
                                     CU_TENSOR_MAP_SWIZZLE_64B);
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
  A.heads_per_item = (kPair || NT == 4) ? 4 : (NT == 1 || !A.two_tiles ? 1 : 2);
  const int max_sq = varlen ? p.max_seqlen_q : p.seqlen_q;
  A.n_qblocks = (max_sq + kBM - 1) / kBM;
  // the softmax works with a positive scale: a negative one negates Q inside
  // the S MMA; a zero scale (uniform weights) becomes a vanishing one
  const float abs_scale = p.softmax_scale < 0.f ? -p.softmax_scale : p.softmax_scale;
  A.scale_log2 = (abs_scale > 0.f ? abs_scale : 1e-30f) * kLog2e;
  A.negate_s = p.softmax_scale < 0.f ? 1u : 0u;
  A.epi = make_epilogue(p.epilogue, p.n_epilogue);
  A.wd = ctx.wd;
  const long long items = static_cast<long long>(A.n_qblocks) * p.batch * (p.hq / A.heads_per_item);
  if (items == 0) return FA_OK;
  if (items > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  auto kern = prefill_tc_kernel<D, kI8, kPair, BN, NT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem) != cudaSuccess)
    return FA_ERR_CUDA;
  note_variant(reinterpret_cast<const void*>(kern));
  if constexpr (kPair) {
    // persistent clusters of two CTAs (one per SM), as many as fit at once
    const int fit = max_pair_clusters(kern, G::kSmem, G::kThreads);
    if (fit <= 0) return FA_ERR_CUDA;
    const long long clusters = items < fit ? items : fit;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    cfg.blockDim = dim3(G::kThreads);
    cfg.dynamicSmemBytes = G::kSmem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tq32, A));
  } else {
    // persistent: one CTA per SM (the shared memory allows no second), each
    // walking its share of the items
    const long long grid = items < device_sm_count() ? items : device_sm_count();
    kern<<<static_cast<unsigned>(grid), G::kThreads, G::kSmem, ctx.stream>>>(tq, tk, tv, tq32, A);
    return cuda_status(cudaGetLastError());
  }
}

// The CTA-pair kernel (one K/V fetch for four heads of a group) serves d =
// 128 when every item's four heads share one KV head (group size a multiple
// of 4) and FA_PREFILL_PAIR=1 (read once).  It is not the default: its
// cross-SM hand-offs (the peer's P to the issuing CTA, completions back)
// lengthen the softmax -> PV -> S chain that bounds this kernel, and it
// measured slower than one CTA per head pair on every workload.
bool use_pair(const fa_fwd_params& p) {
  static const bool enabled = [] {
    const char* e = std::getenv("FA_PREFILL_PAIR");
    return e != nullptr && e[0] == '1';
  }();
  return enabled && p.head_dim == 128 && (p.hq / p.hkv) % 4 == 0;
}

}  // namespace

// d = 64 bf16 with every four consecutive heads in one GQA group: one CTA
// takes four heads (a whole group of four) with 64-key tiles, so four
// softmax tiles share the SM's exponential units and every K/V tile serves
// the four heads.  Selected by FA_PREFILL_QUAD=1 (read once): it measured
// slower than the two-head kernel on the varlen window workload (each
// 64-key step pays the same waits and hand-offs as a 128-key one).
bool use_quad(const fa_fwd_params& p) {
  static const bool enabled = [] {
    const char* e = std::getenv("FA_PREFILL_QUAD");
    return e != nullptr && e[0] == '1';
  }();
  return enabled && p.head_dim == 64 && p.kv_dtype != FA_I8 && (p.hq / p.hkv) % 4 == 0;
}

fa_status launch_prefill_tc(const fa_fwd_params& p, const fa_kv_pages* pages, const RowSink& sink,
                            const LaunchCtx& ctx) {
  const bool pair = use_pair(p);
  if (p.kv_dtype == FA_I8) {
    if (p.head_dim == 128) return pair ? launch_tc<128, true, true>(p, pages, sink, ctx)
                                       : launch_tc<128, true, false>(p, pages, sink, ctx);
    if (p.head_dim == 64) return launch_tc<64, true, false>(p, pages, sink, ctx);
    if (p.head_dim == 32) return launch_tc<32, true, false>(p, pages, sink, ctx);
    if (p.head_dim == 96) return launch_tc<96, true, false>(p, pages, sink, ctx);
    // above 128: one Q tile per CTA, 64-key tiles, separate int8 rings
    if (p.head_dim == 160) return launch_tc<160, true, false, 64, 1>(p, pages, sink, ctx);
    if (p.head_dim == 192) return launch_tc<192, true, false, 64, 1>(p, pages, sink, ctx);
    if (p.head_dim == 224) return launch_tc<224, true, false, 64, 1>(p, pages, sink, ctx);
    if (p.head_dim == 256) return launch_tc<256, true, false, 64, 1>(p, pages, sink, ctx);
    return FA_ERR_UNSUPPORTED;
  }
  if (p.head_dim == 128) return pair ? launch_tc<128, false, true>(p, pages, sink, ctx)
                                     : launch_tc<128, false, false>(p, pages, sink, ctx);
  if (p.head_dim == 64) return use_quad(p) ? launch_tc<64, false, false, 64, 4>(p, pages, sink, ctx)
                                           : launch_tc<64, false, false>(p, pages, sink, ctx);
  if (p.head_dim == 32) return launch_tc<32, false, false>(p, pages, sink, ctx);
  if (p.head_dim == 96) return launch_tc<96, false, false>(p, pages, sink, ctx);
  // above 128: one Q tile per CTA (S of a 64-key tile + O of D columns in TMEM)
  if (p.head_dim == 160) return launch_tc<160, false, false, 64, 1>(p, pages, sink, ctx);
  if (p.head_dim == 192) return launch_tc<192, false, false, 64, 1>(p, pages, sink, ctx);
  if (p.head_dim == 224) return launch_tc<224, false, false, 64, 1>(p, pages, sink, ctx);
  if (p.head_dim == 256) return launch_tc<256, false, false, 64, 1>(p, pages, sink, ctx);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
