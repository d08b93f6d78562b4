// decode.cu -- single-query decode over a KV cache, split along the keys
// (fkl_python PR #6, Verification: a one-query decode step over 256 int8 keys;
// Summary: the kernel dequantises the int8 cache on chip, with no widened
// copy in global memory; kernbench2 commit ADR-0060: decode splits the keys and
// reduces the partial softmax states (m, l, O) to one output).
//
// Work decomposition (stream-K): the 32-key tiles of every (sequence, KV
// head) segment are laid end to end, T tiles in all, and a persistent grid of
// P warps ("workers", 4 per CTA, 2 CTAs per SM; 1 for bf16 at d = 128) takes
// equal contiguous ranges [w*T/P, (w+1)*T/P).  Each worker streams its tiles
// -- K codes, V codes and their fp32 scales -- through its own 3-stage TMA
// ring (128-byte swizzle, bounded mbarrier waits), straight across segment
// boundaries, so the ring never drains and every SM gets the same number of
// bytes.  When a worker's
// range leaves a segment it writes its partial softmax state (m, l, O) for
// the segment's G = hq/hkv query heads to record (segment + worker) and
// counts itself done on the segment; the last worker to finish a segment
// merges its records (the segment's workers are W(x) = (x*P + P - 1) / T
// over its tiles), applies the epilogue and stores bf16.  A one-CTA plan
// kernel first turns the device-side cache lengths into the per-sequence
// tile prefix sums, zeroes the counters and writes the rows of empty caches.
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
// bf16 cache (the same stream-K schedule and merge): tiles arrive as 64-dim
// chunks of 128-byte rows (128-byte swizzle); K fragments come from ldmatrix,
// V^T fragments from ldmatrix.trans, Q enters the bf16 MMA as it is and P is
// rounded to bf16.  A stage is twice as large, so d = 128 runs one CTA per
// SM, and at d = 256 (32 KB for a K and a V tile) each worker's ring holds
// one stage.  Cache rows outside [k_lo, L) may hold any bytes (NaN included): their
// scores are masked, and in a tile that holds such rows the V rows are zeroed
// in shared memory before P V, so 0 * NaN never reaches O.
#include <mutex>
#include <type_traits>

#include "internal.h"

namespace fa {
namespace {

constexpr int kWarps = 4;    // compute warps (workers) per CTA
constexpr int kThreads = (kWarps + 1) * 32;  // plus one producer warp
constexpr int kTile = 32;    // keys per tile
constexpr int kMaxCtasPerSm = 2;  // int8 and bf16 at d = 64; bf16 at d = 128 fits one
constexpr int kMaxWorkers = 4096;
constexpr float kLog2e = 1.4426950408889634f;

struct SkArgs {
  const __nv_bfloat16* q;   // [B*hq, D]
  const float* k_scales;    // [B*hkv, cap]
  const float* v_scales;
  const int32_t* seqlens;   // [B]
  const int32_t* prefix;    // [B+1]: tiles (x hkv) before sequence b; prefix[B] = T (plan kernel)
  int smem_prefix;          // 1: each CTA recomputes the prefix in shared memory (small batches)
  float* rec_o;             // [B*hkv + P][G][D]
  float* rec_ml;            // [B*hkv + P][G][2]
  int32_t* counters;        // [B*hkv]: workers done with each segment (zeroed by the plan)
  __nv_bfloat16* out;       // [B*hq, D]
  Epilogue epi;
  // Groups of more than 8 query heads (the MMA's N) run as kv_split passes
  // over their KV head, each serving group = (hq / hkv_real) / kv_split heads:
  // hkv counts these virtual KV heads (hkv_real * kv_split), and only cache
  // addressing uses the real head g / kv_split.
  int batch, hq, hkv, group, cap, window;
  int hkv_real, kv_split;
  // paged cache (null table: dense [B*hkv, cap, d]): pool [num_pages, hkv,
  // page_size, d]; key j of sequence b lives in page block_table[b*max_pages + j/page_size]
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  int n_workers;            // P (launched warps)
  int min_tiles;            // > 0: at least this many tiles per worker
  float scale_log2;
  Watchdog wd;
};

template <int D, bool kBF>
struct Geom {
  static constexpr int kTileBytes = kTile * D * (kBF ? 2 : 1);  // int8 codes or bf16
  static constexpr int kScaleBytes = kBF ? 0 : 2 * kTile * 4;    // K and V scales (int8)
  static constexpr int kScaleOff = 2 * kTileBytes;
  static constexpr int kStageBytes = ((2 * kTileBytes + kScaleBytes) + 1023) / 1024 * 1024;
  // bf16: 128-byte swizzle of 64-dim chunks [32 rows x 128 B], then for D =
  // 32 or 96 a 32-dim tail chunk [32 rows x 64 B] with the 64-byte swizzle.
  // int8 rows: D = 64 and 128 fill one TMA box with the 64- / 128-byte
  // swizzle; D = 256 is two 128-byte halves (two boxes, 4 KB apart in the
  // tile); D = 32 and 96 are plain rows
  static constexpr int kSwzMask = (kBF || D == 128 || D == 256) ? 0x70 : (D == 64 ? 0x30 : 0);
  static constexpr int kRowBytes = kBF ? 128 : (D > 128 ? 128 : D);  // bytes per row of one box
  static constexpr int kHalves = (!kBF && D > 128) ? D / 128 : 1;   // int8 boxes per tile row
  static constexpr int kChunkBytes = kTile * 128;
  static constexpr int kNFull = D / 64;                 // bf16: full 64-dim chunks
  static constexpr bool kTail = kBF && (D % 64) == 32;  // bf16: a 32-dim tail chunk
  // stages per worker ring (a bf16 tile at D = 256 is 32 KB: one stage,
  // the producer refilling it as soon as its worker releases it)
  static constexpr int kStages = (kBF && D == 256) ? 1 : 3;
  static constexpr int kCtas = ((kBF && (D == 128 || D == 96)) || D == 256) ? 1 : 2;
  static constexpr int kSmem = kWarps * kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  // sequences whose tile prefix fits in the shared memory the CTAs per SM
  // leave over (228 KB per SM, 1 KB reserved per CTA, 256 B margin)
  static constexpr int kPrefixCap = ((233472 / kCtas) - 1024 - kSmem - 256) / 4 - 1;
};
static_assert(Geom<128, true>::kSmem <= 232448, "shared memory budget");
static_assert(2 * Geom<128, false>::kSmem <= 232448 && 2 * Geom<64, false>::kSmem <= 232448 &&
                  2 * Geom<64, true>::kSmem <= 232448,
              "CTAs per SM");
static_assert(Geom<128, false>::kCtas <= kMaxCtasPerSm && Geom<64, true>::kCtas <= kMaxCtasPerSm, "workers");
static_assert(2 * Geom<32, false>::kSmem <= 232448 && 2 * Geom<96, false>::kSmem <= 232448 &&
                  Geom<256, false>::kSmem <= 232448 && Geom<256, true>::kSmem <= 232448 &&
                  2 * Geom<32, true>::kSmem <= 232448 &&
                  Geom<96, true>::kSmem <= 232448,
              "CTAs per SM");

// TMA swizzle of a byte offset inside a tile whose base is aligned to the
// swizzle period: bits [4,7) (128B) or [4,6) (64B) ^= bits [7,10) / [7,9).
template <int D, bool kBF>
__device__ __forceinline__ uint32_t swz(uint32_t lin) {
  return lin ^ ((lin >> 3) & Geom<D, kBF>::kSwzMask);
}
// Offset of byte b of int8 row r inside a tile (the box halves of D = 256).
template <int D>
__device__ __forceinline__ uint32_t i8_off(int r, int b) {
  using G = Geom<D, false>;
  return (b / G::kRowBytes) * (kTile * G::kRowBytes) + swz<D, false>(r * G::kRowBytes + b % G::kRowBytes);
}
// Shared address of element (key r, dim c) of a bf16 tile at `tile`.
template <int D>
__device__ __forceinline__ uint32_t bf_addr(uint32_t tile, int r, int c) {
  using G = Geom<D, true>;
  if (G::kTail && c / 64 == G::kNFull) {  // the 32-dim tail: 64-byte rows, 64-byte swizzle
    const uint32_t lin = r * 64 + (c % 64) * 2;
    return tile + G::kNFull * G::kChunkBytes + (lin ^ ((lin >> 3) & 0x30));
  }
  return tile + (c / 64) * G::kChunkBytes + swz<D, true>(r * 128 + (c % 64) * 2);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
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

// fp16x2 pairs 1152 + c of the signed bytes of w: bytes 0, 2 -> even and
// 1, 3 -> odd (exact; the caller removes the bias).  byte ^ 0x80 = c + 128
// becomes the low mantissa byte of 1024 (fp16 0x6400).
__device__ __forceinline__ void i8x4_to_f16x2_biased(uint32_t w, uint32_t& even, uint32_t& odd) {
  const uint32_t x = w ^ 0x80808080u;
  even = prmt(x, 0x64646464u, 0x4240);
  odd = prmt(x, 0x64646464u, 0x4341);
}
constexpr float kCodeBias = 1152.0f;

// Four 8x8 b16 matrices; lane l gives the row address of matrix l / 8, row l % 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}


__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
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
__host__ __device__ __forceinline__ void key_range(int L, int window, int& k_lo, int& t_begin) {
  k_lo = window > 0 ? (L - window > 0 ? L - window : 0) : 0;
  t_begin = (k_lo / kTile) * kTile;
}
__device__ __forceinline__ int clamp_len(int L, int cap) { return max(0, min(L, cap)); }
__device__ __forceinline__ int tiles_of(int L, int window) {
  int k_lo, t_begin;
  key_range(L, window, k_lo, t_begin);
  return L > t_begin ? (L - t_begin + kTile - 1) / kTile : 0;
}

// Programmatic dependent launch: the plan kernel lets the decode kernel
// start at once; the decode kernel waits for the plan's completion (its
// zeroed counters) only where it first needs them.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// The worker whose range [w*T/P, (w+1)*T/P) holds tile x.
__device__ __forceinline__ int worker_of(long long x, long long T, long long P) {
  return static_cast<int>((x * P + P - 1) / T);
}
__device__ __forceinline__ long long worker_begin(long long w, long long T, long long P) { return (w * T) / P; }
// Never more workers than tiles, so every worker's range is non-empty and a
// segment's workers are exactly W(first tile) .. W(last tile).
__device__ __forceinline__ int effective_workers(const SkArgs& A, long long T) {
  long long p = min(static_cast<long long>(A.n_workers), max(1LL, T));
  if (A.min_tiles > 0) p = min(p, max(1LL, T / A.min_tiles));
  return static_cast<int>(p);
}

// ---------------------------------------------------------------- plan
// prefix[b] = sum over earlier sequences of (tiles x hkv); prefix[B] = T.
// A length outside [0, cap] is clamped (every kernel of the call clamps it
// the same way) and reported in the status word.
template <int D>
__global__ void __launch_bounds__(1024) decode_plan_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                           int hq, int hkv, int cap, int window,
                                                           int32_t* __restrict__ prefix,
                                                           int32_t* __restrict__ counters,
                                                           __nv_bfloat16* __restrict__ out, Epilogue epi,
                                                           unsigned int* status) {
  griddep_launch_dependents();
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;
  const int per = (batch + nthreads - 1) / nthreads;
  const int b0 = min(batch, tid * per), b1 = min(batch, b0 + per);
  int32_t local = 0;
  bool bad = false;
  for (int b = b0; b < b1; ++b) {
    const int L = seqlens[b];
    bad |= L < 0 || L > cap;
    local += tiles_of(clamp_len(L, cap), window) * hkv;
  }
  if (bad) atomicOr(status, kStatusRange);
  int32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t v = lane < (nthreads >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    warp_sums[lane] = v;
  }
  __syncthreads();
  int32_t base = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - local;
  for (int b = b0; b < b1; ++b) {
    prefix[b] = base;
    const int tb = tiles_of(clamp_len(seqlens[b], cap), window);
    base += tb * hkv;
    if (tb == 0) {
      // a sequence with no key to attend: the epilogue of zeros (no worker
      // sees it); rare, so one thread writes its rows
      const __nv_bfloat16 zero_row = __float2bfloat16_rn(apply_epilogue(0.f, epi));
      for (int i = 0; i < hq * D; ++i) out[static_cast<int64_t>(b) * hq * D + i] = zero_row;
    }
  }
  if (tid == nthreads - 1) prefix[batch] = base;
  for (int i = tid; i < batch * hkv; i += nthreads) counters[i] = 0;
}

// Position in the global tile sequence: sequence b, KV head g, tile t of Tb,
// with the segment's first tile key and cache row kept for the loads.
struct Cursor {
  int b, g, t, Tb;
  int t_begin;      // key of the segment's first tile
  int64_t kv_row0;  // cache row of key 0 of (b, g)
};

__device__ __forceinline__ int seq_tiles(const SkArgs& A, const int32_t* pre, int b) {
  return (pre[b + 1] - pre[b]) / A.hkv;
}
__device__ __forceinline__ void set_segment(const SkArgs& A, Cursor& c) {
  int k_lo;
  key_range(clamp_len(A.seqlens[c.b], A.cap), A.window, k_lo, c.t_begin);
  c.kv_row0 = (static_cast<int64_t>(c.b) * A.hkv_real + c.g / A.kv_split) * A.cap;
}
__device__ __forceinline__ Cursor locate(const SkArgs& A, const int32_t* pre, long long x) {
  int lo = 0, hi = A.batch - 1;  // largest b with prefix[b] <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= x) lo = mid; else hi = mid - 1;
  }
  Cursor c;
  c.b = lo;
  c.Tb = seq_tiles(A, pre, lo);
  const long long y = x - pre[lo];
  c.g = static_cast<int>(y / c.Tb);
  c.t = static_cast<int>(y % c.Tb);
  set_segment(A, c);
  return c;
}
__device__ __forceinline__ void advance(const SkArgs& A, const int32_t* pre, Cursor& c) {
  if (++c.t < c.Tb) return;
  c.t = 0;
  if (++c.g < A.hkv) {
    c.kv_row0 += A.cap;
    return;
  }
  c.g = 0;
  do {
    ++c.b;
  } while (c.b < A.batch && (c.Tb = seq_tiles(A, pre, c.b)) == 0);
  if (c.b < A.batch) set_segment(A, c);
}

// Cache row of the 32-key tile starting at key0 of segment (c.b, c.g).  For a
// paged cache the issuing lane keeps the page of its current (sequence,
// logical page) -- every KV head of a sequence shares it, and a page spans
// page_size / 32 tiles -- and loads the next page's id as soon as it enters
// a page, so the table read is off the issue path.  A page id outside the
// pool is reported and replaced by page 0, so no load leaves the pool (that
// sequence's result is then meaningless).
struct PageCursor {
  int b = -1, lp = -1, pg = 0, next = -1;
};
__device__ __forceinline__ int page_id(const SkArgs& A, int b, int lp) {
  return lp < A.max_pages ? __ldg(A.block_table + static_cast<int64_t>(b) * A.max_pages + lp) : 0;
}
__device__ __forceinline__ int64_t tile_row(const SkArgs& A, const Cursor& c, int key0, PageCursor& pc) {
  if (A.block_table == nullptr) return c.kv_row0 + key0;
  const int lp = key0 / A.page_size;
  if (c.b != pc.b || lp != pc.lp) {
    int pg = (c.b == pc.b && lp == pc.lp + 1) ? pc.next : page_id(A, c.b, lp);
    if (pg < 0 || pg >= A.num_pages) {
      record_status(A.wd, kStatusRange);
      pg = 0;
    }
    pc.b = c.b;
    pc.lp = lp;
    pc.pg = pg;
    pc.next = page_id(A, c.b, lp + 1);  // consumed page_size / 32 tiles later
  }
  return (static_cast<int64_t>(pc.pg) * A.hkv_real + c.g / A.kv_split) * A.page_size + key0 % A.page_size;
}

template <int D, bool kBF>
__global__ void __launch_bounds__(kThreads, Geom<D, kBF>::kCtas)
    decode_sk_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_k32, const __grid_constant__ CUtensorMap tm_v32,
                     const SkArgs A) {
  using G = Geom<D, kBF>;
  constexpr int kStages = G::kStages;
  constexpr int kSteps = D / 16;      // k-steps of the S MMA
  constexpr int kChunks = D / 64;     // 16-byte chunks per thread per K row (d = 64, 128)
  // d = 64 and 128: thread qq owns dims [qq D/4, (qq+1) D/4) of every K row
  // (16-byte loads); other head sizes: dims [32 c + 8 qq, +8) of every 32-dim
  // block c (8-byte loads).  Either way k-step ks reads one 4-byte word of
  // the thread's dims, and Q's fragments take the same dims in that order.
  constexpr bool kQuarter = (D == 64 || D == 128);
  constexpr int kMT = D / 16;         // O^T m-tiles (dims)
  extern __shared__ uint8_t dec_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * G::kStageBytes);
  __shared__ int abort_flag;

  // full[w][s]: the producer's TMA landed stage s of worker w's ring;
  // empty[w][s]: worker w is done reading it
  uint64_t* empty_bars = bars + kWarps * kStages;
  int32_t* s_pre = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + 256);
  __shared__ int32_t warp_sums[kWarps + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qq = lane & 3;
  if (threadIdx.x == 0) abort_flag = 0;
  if (warp < kWarps && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[warp * kStages + s], 1);
      mbar_init(&empty_bars[warp * kStages + s], 1);
    }
    fence_barrier_init();
  }
  // the tile prefix over sequences: computed here for small batches (no
  // dependence on the plan kernel until the first counter), else the plan's
  const int32_t* pre = A.prefix;
  if (A.smem_prefix) {
    int32_t carry = 0;
    for (int b0 = 0; b0 < A.batch; b0 += kThreads) {
      const int b = b0 + static_cast<int>(threadIdx.x);
      const int32_t own = b < A.batch ? tiles_of(clamp_len(A.seqlens[b], A.cap), A.window) * A.hkv : 0;
      int32_t incl = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (lane == 31) warp_sums[warp] = incl;
      __syncthreads();
      int32_t before = carry;
      for (int v = 0; v < warp; ++v) before += warp_sums[v];
      if (b < A.batch) s_pre[b] = before + incl - own;
      for (int v = warp; v < kWarps + 1; ++v) before += warp_sums[v];
      carry = before;  // the same in every thread: the running total
      __syncthreads();
    }
    if (threadIdx.x == 0) s_pre[A.batch] = carry;
    pre = s_pre;
  } else {
    griddep_wait();
  }
  __syncthreads();

  const long long T = pre[A.batch];
  const long long P = effective_workers(A, T);
  if (warp == kWarps) {
    // ---------------------------------------------------------------- producer
    // Lanes 0 .. kWarps-1 keep the workers' rings full, lane l for worker l
    // with that worker's own cursor.  The lanes run together: each round,
    // every lane whose next stage its worker has released (a non-blocking
    // probe) refills it, so up to four refills share one pass of the issue
    // code and no load issue sits in a compute warp.  Gives up (status word)
    // when no ring frees a stage for a whole watchdog budget.
    if (T == 0) return;
    const long long wl = static_cast<long long>(blockIdx.x) * kWarps + lane;
    int n = 0;
    Cursor ic;
    PageCursor ipc;
    if (lane < kWarps && wl < P) {
      const long long tf = worker_begin(wl, T, P);
      n = static_cast<int>(worker_begin(wl + 1, T, P) - tf);
      ic = locate(A, pre, tf);
    }
    int i = 0;
    long long t0 = clock64();
    while (__any_sync(0xffffffffu, i < n)) {
      const int s = i % kStages;
      const bool ready = i < n && (i < kStages ||
                                   mbar_test_wait(smem_u32(&empty_bars[lane * kStages + s]), ((i / kStages) - 1) & 1));
      if (ready) {
        const int key0 = ic.t_begin + ic.t * kTile;
        const int64_t row = tile_row(A, ic, key0, ipc);
        uint8_t* st = smem + (lane * kStages + s) * G::kStageBytes;
        uint64_t* bar = &bars[lane * kStages + s];
        mbar_expect_tx(bar, 2 * G::kTileBytes + G::kScaleBytes);
        if constexpr (kBF) {
#pragma unroll
          for (int c = 0; c < G::kNFull; ++c) {
            tma_load_2d(st + c * G::kChunkBytes, &tm_k, bar, 64 * c, static_cast<int>(row));
            tma_load_2d(st + G::kTileBytes + c * G::kChunkBytes, &tm_v, bar, 64 * c, static_cast<int>(row));
          }
          if constexpr (G::kTail) {
            tma_load_2d(st + G::kNFull * G::kChunkBytes, &tm_k32, bar, 64 * G::kNFull, static_cast<int>(row));
            tma_load_2d(st + G::kTileBytes + G::kNFull * G::kChunkBytes, &tm_v32, bar, 64 * G::kNFull,
                        static_cast<int>(row));
          }
        } else {
#pragma unroll
          for (int h = 0; h < G::kHalves; ++h) {
            tma_load_2d(st + h * kTile * G::kRowBytes, &tm_k, bar, G::kRowBytes * h, static_cast<int>(row));
            tma_load_2d(st + G::kTileBytes + h * kTile * G::kRowBytes, &tm_v, bar, G::kRowBytes * h,
                        static_cast<int>(row));
          }
          bulk_load(st + G::kScaleOff, A.k_scales + row, kTile * 4, bar);
          bulk_load(st + G::kScaleOff + kTile * 4, A.v_scales + row, kTile * 4, bar);
        }
        advance(A, pre, ic);
        ++i;
      }
      if (__any_sync(0xffffffffu, ready)) {
        t0 = clock64();
      } else if (clock64() - t0 > A.wd.budget) {
        if (lane == 0) record_status(A.wd, kStatusTimeout);
        return;
      } else {
        __nanosleep(32);  // leave the issue slots of this sub-partition to its worker
      }
    }
    return;
  }
  const long long w = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (T == 0 || w >= P) return;
  const long long t_first = worker_begin(w, T, P);
  const int my_tiles = static_cast<int>(worker_begin(w + 1, T, P) - t_first);
  if (my_tiles <= 0) return;

  auto stage_ptr = [&](int s) { return smem + (warp * kStages + s) * G::kStageBytes; };
  // ---- per-segment state
  uint32_t qb0[kSteps], qb1[kSteps];
  float qs0 = 0.f, qs1 = 0.f;
  float cb0 = 0.f, cb1 = 0.f;  // int8: 1152 * sum of the (prescaled fp16) q of heads 2qq, 2qq+1
  float o[kMT][4];
  float m_run[2], l_run[2];
  auto reset = [&]() {
#pragma unroll
    for (int m = 0; m < kMT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  };
  // Q fragments: thread (gq, qq) holds head gq, dims [qq*D/4, (qq+1)*D/4)
  auto load_q = [&](int b, int g) {
    const bool head_ok = gq < A.group;
    const int hq_idx = b * A.hq + g * A.group + gq;
    if constexpr (kBF) {
      // B fragments of head gq: dims 16 ks + 2 qq (+1) and 16 ks + 8 + 2 qq (+1)
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(A.q + static_cast<int64_t>(hq_idx) * D);
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        qb0[ks] = head_ok ? qw[8 * ks + qq] : 0u;
        qb1[ks] = head_ok ? qw[8 * ks + 4 + qq] : 0u;
      }
      qs0 = qs1 = A.scale_log2;
      return;
    }
    float qv[D / 4];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint4 raw = make_uint4(0, 0, 0, 0);
      const int dim0 = kQuarter ? qq * (D / 4) + 8 * c : 32 * c + 8 * qq;
      if (head_ok) raw = *reinterpret_cast<const uint4*>(A.q + static_cast<int64_t>(hq_idx) * D + dim0);
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[8 * c + 2 * e] = __uint_as_float(wv[e] << 16);
        qv[8 * c + 2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < D / 4; ++e) amax = fmaxf(amax, fabsf(qv[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);
    const int kexp = amax > 0.f ? 15 - ex : 0;  // largest |q| * 2^kexp in [2^14, 2^15)
    const float qs_own = ldexpf(A.scale_log2, -kexp);
    // K codes enter the MMA as 1152 + c, so every score of head n carries
    // 1152 * (sum over dims of its fp16 q); the sum of these fp16 values is
    // exact in fp64
    double qsum = 0.0;
#pragma unroll
    for (int ks = 0; ks < kSteps; ++ks) {
      qb0[ks] = pack_f16x2(ldexpf(qv[4 * ks + 0], kexp), ldexpf(qv[4 * ks + 2], kexp));
      qb1[ks] = pack_f16x2(ldexpf(qv[4 * ks + 1], kexp), ldexpf(qv[4 * ks + 3], kexp));
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&qb0[ks]));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&qb1[ks]));
      qsum += (static_cast<double>(f0.x) + f0.y) + (static_cast<double>(f1.x) + f1.y);
    }
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
    const float cb_own = static_cast<float>(qsum * static_cast<double>(kCodeBias));
    // logit multipliers and biases of this thread's two score columns (heads 2qq, 2qq+1)
    qs0 = __shfl_sync(0xffffffffu, qs_own, (2 * qq) * 4);
    qs1 = __shfl_sync(0xffffffffu, qs_own, (2 * qq + 1) * 4);
    cb0 = __shfl_sync(0xffffffffu, cb_own, (2 * qq) * 4);
    cb1 = __shfl_sync(0xffffffffu, cb_own, (2 * qq + 1) * 4);
  };
  // partial state of segment `seg` -> record (seg + w)
  auto finalize = [&](int seg) {
    float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int64_t rec = static_cast<int64_t>(seg) + w;
    const int h0 = 2 * qq, h1 = 2 * qq + 1;
    if (gq == 0) {
      if (h0 < A.group) {
        A.rec_ml[(rec * A.group + h0) * 2 + 0] = m_run[0];
        A.rec_ml[(rec * A.group + h0) * 2 + 1] = l0;
      }
      if (h1 < A.group) {
        A.rec_ml[(rec * A.group + h1) * 2 + 0] = m_run[1];
        A.rec_ml[(rec * A.group + h1) * 2 + 1] = l1;
      }
    }
    if constexpr (kBF) {
      // m-tile mi holds dims 16 mi + gq (c0, c1) and 16 mi + gq + 8 (c2, c3)
#pragma unroll
      for (int mi = 0; mi < kMT; ++mi) {
        const int dim = 16 * mi + gq;
        if (h0 < A.group) {
          A.rec_o[(rec * A.group + h0) * D + dim] = o[mi][0];
          A.rec_o[(rec * A.group + h0) * D + dim + 8] = o[mi][2];
        }
        if (h1 < A.group) {
          A.rec_o[(rec * A.group + h1) * D + dim] = o[mi][1];
          A.rec_o[(rec * A.group + h1) * D + dim + 8] = o[mi][3];
        }
      }
    } else {
#pragma unroll
      for (int pr = 0; pr < D / 32; ++pr) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int dim0 = 4 * (8 * pr + gq) + 2 * j;
          const float(&c)[4] = o[2 * pr + j];
          if (h0 < A.group)
            *reinterpret_cast<float2*>(A.rec_o + (rec * A.group + h0) * D + dim0) = make_float2(c[0], c[2]);
          if (h1 < A.group)
            *reinterpret_cast<float2*>(A.rec_o + (rec * A.group + h1) * D + dim0) = make_float2(c[1], c[3]);
        }
      }
    }
  };

  // The last worker done with a segment merges every record of it.
  auto segment_workers = [&](int seg, int& w_lo, int& w_hi) {
    const int b = seg / A.hkv, g = seg % A.hkv;
    const int Tb = seq_tiles(A, pre, b);
    const long long a = pre[b] + static_cast<long long>(g) * Tb;
    w_lo = worker_of(a, T, P);
    w_hi = worker_of(a + Tb - 1, T, P);
  };
  auto finish = [&](int seg) {
    finalize(seg);
    __threadfence();  // each lane's record stores are visible device-wide ...
    __syncwarp();     // ... before lane 0 counts the warp done
    int prev = 0;
    if (lane == 0) {
      griddep_wait();  // the plan kernel has zeroed the counters
      prev = atomicAdd(&A.counters[seg], 1);
    }
    prev = __shfl_sync(0xffffffffu, prev, 0);
    int w_lo, w_hi;
    segment_workers(seg, w_lo, w_hi);
    if (prev != w_hi - w_lo) return;
    __threadfence();
    const int b = seg / A.hkv, g = seg % A.hkv;
    // one pass over the segment's records with an online max; lane l owns
    // head l / 4 and a quarter of its dims (contiguous, read as float4), and
    // the unrolled record loop keeps several records' loads in flight
    constexpr int kPer = D / 4;
    const int hl = lane >> 2, part = lane & 3;
    if (hl < A.group) {
      float M = -INFINITY, lsum = 0.f, acc[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
#pragma unroll 2
      for (int v = w_lo; v <= w_hi; ++v) {
        const int64_t r = (static_cast<int64_t>(seg) + v) * A.group + hl;
        const float m = __ldcg(&A.rec_ml[r * 2]);
        const float lv = __ldcg(&A.rec_ml[r * 2 + 1]);
        const float4* src = reinterpret_cast<const float4*>(A.rec_o + r * D + part * kPer);
        float4 ov[kPer / 4];
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) ov[q] = __ldcg(src + q);
        const float mn = fmaxf(M, m);
        const float ref = mn == -INFINITY ? 0.f : mn;
        const float a_old = ex2_approx(M - ref), a_new = ex2_approx(m - ref);
        M = mn;
        lsum = lsum * a_old + lv * a_new;
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
          acc[4 * q + 0] = acc[4 * q + 0] * a_old + ov[q].x * a_new;
          acc[4 * q + 1] = acc[4 * q + 1] * a_old + ov[q].y * a_new;
          acc[4 * q + 2] = acc[4 * q + 2] * a_old + ov[q].z * a_new;
          acc[4 * q + 3] = acc[4 * q + 3] * a_old + ov[q].w * a_new;
        }
      }
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int j = 0; j < kPer; ++j) acc[j] *= inv;
      apply_epilogue_vec(acc, A.epi);
      uint4* dst = reinterpret_cast<uint4*>(A.out + (static_cast<int64_t>(b) * A.hq + g * A.group + hl) * D +
                                            part * kPer);
#pragma unroll
      for (int q = 0; q < kPer / 8; ++q)
        dst[q] = make_uint4(pack_bf16x2(acc[8 * q + 0], acc[8 * q + 1]), pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]),
                            pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]), pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]));
    }
  };

  Cursor cc = locate(A, pre, t_first);
  int cur_seg = -1;
  int seg_t_begin = 0, k_lo = 0, key_end = 0;
  for (int i = 0; i < my_tiles; ++i) {
    const int seg = cc.b * A.hkv + cc.g;
    if (seg != cur_seg) {
      if (cur_seg >= 0) finish(cur_seg);
      reset();
      load_q(cc.b, cc.g);
      cur_seg = seg;
      key_end = clamp_len(A.seqlens[cc.b], A.cap);
      key_range(key_end, A.window, k_lo, seg_t_begin);
    }
    const int key0 = seg_t_begin + cc.t * kTile;

    const int s = i % kStages;
    // every lane polls; the decision to continue is warp-uniform because the
    // MMAs and transposes below need the whole warp
    const bool ready = wait_parity(&bars[warp * kStages + s], (i / kStages) & 1, A.wd, &abort_flag);
    if (!__all_sync(0xffffffffu, ready)) break;
    const uint32_t kt = smem_u32(stage_ptr(s));
    const uint32_t vt = kt + G::kTileBytes;
    const float* ksc = reinterpret_cast<const float*>(stage_ptr(s) + G::kScaleOff);
    const float* vsc = ksc + kTile;

    // ---- S^T = K . Q^T for the two 16-key halves of the tile
    float sc[2][4];
    if constexpr (kBF) {
      // matrix i of lane l: keys 16 mt + 8 (i % 2) + l % 8, dims 16 ks + 8 (i / 2)
      const int mi = lane >> 3, mr = lane & 7;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < kSteps; ++ks) {
          uint32_t a[4];
          ldsm_x4(bf_addr<D>(kt, 16 * mt + 8 * (mi % 2) + mr, 16 * ks + 8 * (mi / 2)), a);
          mma16816_bf16(sc[mt], a, qb0[ks], qb1[ks]);
        }
      }
    } else
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
      const int r0 = 16 * mt + gq, r1 = r0 + 8;
      // this thread's K words of rows r0, r1: word ks feeds k-step ks
      uint32_t kwa[kSteps], kwb[kSteps];
      if constexpr (kQuarter) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const uint32_t off = (qq * kChunks + c) * 16;
          const uint4 a4 = lds128(kt + swz<D, false>(r0 * D + off));
          const uint4 b4 = lds128(kt + swz<D, false>(r1 * D + off));
          kwa[4 * c] = a4.x; kwa[4 * c + 1] = a4.y; kwa[4 * c + 2] = a4.z; kwa[4 * c + 3] = a4.w;
          kwb[4 * c] = b4.x; kwb[4 * c + 1] = b4.y; kwb[4 * c + 2] = b4.z; kwb[4 * c + 3] = b4.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint2 a2 = lds64(kt + i8_off<D>(r0, 32 * c + 8 * qq));
          const uint2 b2 = lds64(kt + i8_off<D>(r1, 32 * c + 8 * qq));
          kwa[2 * c] = a2.x; kwa[2 * c + 1] = a2.y;
          kwb[2 * c] = b2.x; kwb[2 * c + 1] = b2.y;
        }
      }
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        const uint32_t wa = kwa[ks];
        const uint32_t wb = kwb[ks];
        uint32_t ae, ao, be, bo;
        i8x4_to_f16x2_biased(wa, ae, ao);
        i8x4_to_f16x2_biased(wb, be, bo);
        mma16816(sc[mt], ae, be, ao, bo, qb0[ks], qb1[ks]);
      }
    }

    // ---- online softmax (per head column); only a tile that reaches past
    // the band's ends masks by key position (warp-uniform choice)
    uint32_t pb[2][2];  // [mt][b0/b1] P' operand fragments
    auto softmax = [&](auto masked_tag) {
      constexpr bool kMasked = decltype(masked_tag)::value;
      float x[2][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int kl = 16 * mt + gq + 8 * hf;
          const int key = key0 + kl;
          const bool ok = !kMasked || (key >= k_lo && key < key_end);
          float x0, x1;
          if constexpr (kBF) {
            x0 = sc[mt][2 * hf + 0] * qs0;
            x1 = sc[mt][2 * hf + 1] * qs1;
          } else {
            const float kscale = ksc[kl];
            x0 = (sc[mt][2 * hf + 0] - cb0) * (kscale * qs0);
            x1 = (sc[mt][2 * hf + 1] - cb1) * (kscale * qs1);
          }
          x[mt][2 * hf + 0] = ok ? x0 : -INFINITY;
          x[mt][2 * hf + 1] = ok ? x1 : -INFINITY;
          mx0 = fmaxf(mx0, x[mt][2 * hf + 0]);
          mx1 = fmaxf(mx1, x[mt][2 * hf + 1]);
        }
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      // the running maxima move only when a tile raises them, and the O
      // rescale runs only when some head of the warp moved
      const bool up0 = mx0 > m_run[0], up1 = mx1 > m_run[1];
      if (__any_sync(0xffffffffu, up0 || up1)) {
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float r0 = mn0 == -INFINITY ? 0.f : mn0, r1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = ex2_approx(m_run[0] - r0), al1 = ex2_approx(m_run[1] - r1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        l_run[0] *= al0;
        l_run[1] *= al1;
#pragma unroll
        for (int m = 0; m < kMT; ++m) {
          o[m][0] *= al0; o[m][2] *= al0;
          o[m][1] *= al1; o[m][3] *= al1;
        }
      }
      const float ref0 = m_run[0] == -INFINITY ? 0.f : m_run[0];
      const float ref1 = m_run[1] == -INFINITY ? 0.f : m_run[1];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        uint32_t packed[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int kl = 16 * mt + gq + 8 * hf;
          const int key = key0 + kl;
          const bool ok = !kMasked || (key >= k_lo && key < key_end);
          const float p0 = ex2_approx(x[mt][2 * hf + 0] - ref0);
          const float p1 = ex2_approx(x[mt][2 * hf + 1] - ref1);
          l_run[0] += p0;
          l_run[1] += p1;
          if constexpr (kBF) {
            packed[hf] = kMasked ? pack_bf16x2(ok ? p0 : 0.f, ok ? p1 : 0.f) : pack_bf16x2(p0, p1);
          } else {
            const float vscale = ok ? vsc[kl] : 0.f;
            packed[hf] = pack_f16x2(p0 * vscale, p1 * vscale);
          }
        }
        pb[mt][0] = transpose8x8(packed[0]);  // (head gq; keys 2qq, 2qq+1)
        pb[mt][1] = transpose8x8(packed[1]);  // (head gq; keys 8+2qq, 8+2qq+1)
      }
    };
    const bool interior = key0 >= k_lo && key0 + kTile <= key_end;
    if (interior) {
      softmax(std::false_type{});
    } else {
      softmax(std::true_type{});
    }

    // ---- O^T += V^T . P'
    if constexpr (kBF) {
      if (key0 < k_lo || key0 + kTile > key_end) {
        // rows outside the band may hold NaN or Inf: zero them (P is 0 there)
        const int key = key0 + lane;
        if (key < k_lo || key >= key_end) {
#pragma unroll
          for (int c = 0; c < D; c += 8)
            asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(bf_addr<D>(vt, lane, c)), "r"(0u) : "memory");
          fence_proxy_async_smem();  // ordered before the TMA that refills this stage
        }
        __syncwarp();
      }
      // matrix i of lane l: keys 16 mt + 8 (i / 2) + l % 8, dims 16 mi + 8 (i % 2)
      const int mi4 = lane >> 3, mr = lane & 7;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int mi = 0; mi < kMT; ++mi) {
          uint32_t a[4];
          ldsm_x4_trans(bf_addr<D>(vt, 16 * mt + 8 * (mi4 / 2) + mr, 16 * mi + 8 * (mi4 % 2)), a);
          mma16816_bf16(o[mi], a, pb[mt][0], pb[mt][1]);
        }
      }
    } else
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int kk0 = 16 * mt + 2 * qq;
#pragma unroll
      for (int pr = 0; pr < D / 32; ++pr) {
        const uint32_t xw = (8 * pr + gq) * 4;  // byte offset of this thread's word
        const uint32_t w0 = lds32(vt + i8_off<D>(kk0 + 0, xw));
        const uint32_t w1 = lds32(vt + i8_off<D>(kk0 + 1, xw));
        const uint32_t w2 = lds32(vt + i8_off<D>(kk0 + 8, xw));
        const uint32_t w3 = lds32(vt + i8_off<D>(kk0 + 9, xw));
        const uint32_t t01l = prmt(w0, w1, 0x5410), t01h = prmt(w0, w1, 0x7632);
        const uint32_t t23l = prmt(w2, w3, 0x5410), t23h = prmt(w2, w3, 0x7632);
        mma16816(o[2 * pr], i8x2_to_f16x2_even(t01l), i8x2_to_f16x2_odd(t01l), i8x2_to_f16x2_even(t23l),
                 i8x2_to_f16x2_odd(t23l), pb[mt][0], pb[mt][1]);
        mma16816(o[2 * pr + 1], i8x2_to_f16x2_even(t01h), i8x2_to_f16x2_odd(t01h),
                 i8x2_to_f16x2_even(t23h), i8x2_to_f16x2_odd(t23h), pb[mt][0], pb[mt][1]);
      }
    }

    // this warp is done with the stage: hand it back to the producer
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive(&empty_bars[warp * kStages + s]);
    }
    advance(A, pre, cc);
  }
  if (cur_seg >= 0) finish(cur_seg);
}

// plan (prefix [B+1]) and counters [B*hkv <= B*hq], 256-byte padded
size_t plan_bytes(int batch, int hq) {
  return (static_cast<size_t>(batch + 1 + static_cast<size_t>(batch) * hq) * sizeof(int32_t) + 255) / 256 * 256;
}
size_t records_bytes(int batch, int hq, int hkv, int d, int n_workers) {
  const size_t recs = static_cast<size_t>(batch) * hkv + n_workers;
  return recs * (hq / hkv) * (static_cast<size_t>(d) + 2) * sizeof(float);
}

// Launch plan + stream-K kernel + merge into `ws` (plan, then records).
template <int D, bool kBF>
fa_status launch_sk(const fa_decode_params& p, const fa_kv_pages* pages, int n_workers, int min_tiles, void* ws,
                    bool count_variants, const LaunchCtx& ctx) {
  using G = Geom<D, kBF>;
  const uint64_t rows = pages != nullptr
                            ? static_cast<uint64_t>(pages->num_pages) * p.hkv * pages->page_size
                            : static_cast<uint64_t>(p.batch) * p.hkv * p.capacity;
  CUtensorMap tmk, tmv;
  const uint64_t dims[2] = {static_cast<uint64_t>(D), rows};
  const uint64_t strides[1] = {static_cast<uint64_t>(D) * (kBF ? 2 : 1)};
  // int8: one box of whole rows; bf16: boxes of 64 dims (128 bytes) per row
  // bf16: boxes of 64 dims (128 bytes) per row; int8: boxes of G::kRowBytes
  const uint32_t box[2] = {static_cast<uint32_t>(kBF ? 64 : G::kRowBytes), static_cast<uint32_t>(kTile)};
  const CUtensorMapSwizzle sw = G::kSwzMask == 0x70   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : G::kSwzMask == 0x30 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUtensorMapDataType dt = kBF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  fa_status st = encode_tensor_map(&tmk, dt, 2, p.k_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;
  st = encode_tensor_map(&tmv, dt, 2, p.v_cache, dims, strides, box, sw);
  if (st != FA_OK) return st;
  CUtensorMap tmk32 = tmk, tmv32 = tmv;  // bf16 32-dim tails: boxes of 32 dims, 64-byte swizzle
  if constexpr (G::kTail) {
    const uint32_t box32[2] = {32, static_cast<uint32_t>(kTile)};
    st = encode_tensor_map(&tmk32, dt, 2, p.k_cache, dims, strides, box32, CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != FA_OK) return st;
    st = encode_tensor_map(&tmv32, dt, 2, p.v_cache, dims, strides, box32, CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != FA_OK) return st;
  }

  // a group of G > 8 query heads runs as `split` passes of G / split <= 8
  const int full_group = p.hq / p.hkv;
  int split = (full_group + 7) / 8;
  while (full_group % split != 0) ++split;
  const int group = full_group / split;
  const int hkv = p.hkv * split;
  uint8_t* base = static_cast<uint8_t*>(ws);
  SkArgs A;
  A.q = static_cast<const __nv_bfloat16*>(p.q);
  A.k_scales = p.k_scales;
  A.v_scales = p.v_scales;
  A.seqlens = p.cache_seqlens;
  A.prefix = reinterpret_cast<int32_t*>(base);
  A.counters = reinterpret_cast<int32_t*>(base) + (p.batch + 1);
  A.out = static_cast<__nv_bfloat16*>(p.out);
  A.epi = make_epilogue(p.epilogue, p.n_epilogue);
  const size_t o_recs = static_cast<size_t>(p.batch * hkv + n_workers) * group;
  A.rec_o = reinterpret_cast<float*>(base + plan_bytes(p.batch, p.hq));
  A.rec_ml = A.rec_o + o_recs * D;
  A.batch = p.batch;
  A.hq = p.hq;
  A.hkv = hkv;
  A.group = group;
  A.hkv_real = p.hkv;
  A.kv_split = split;
  A.cap = p.capacity;
  A.block_table = pages != nullptr ? pages->block_table : nullptr;
  A.max_pages = pages != nullptr ? pages->max_pages : 1;
  A.page_size = pages != nullptr ? pages->page_size : p.capacity;
  A.num_pages = pages != nullptr ? pages->num_pages : p.batch;
  A.window = p.window;
  A.n_workers = n_workers;
  A.min_tiles = min_tiles;
  A.scale_log2 = p.softmax_scale * kLog2e;
  A.wd = ctx.wd;

  auto plan = decode_plan_kernel<D>;
  auto kern = decode_sk_kernel<D, kBF>;
  if (count_variants) {
    note_variant(reinterpret_cast<const void*>(plan));
    note_variant(reinterpret_cast<const void*>(kern));
  }
  plan<<<1, 1024, 0, ctx.stream>>>(p.cache_seqlens, p.batch, p.hq, hkv, p.capacity, p.window,
                                   reinterpret_cast<int32_t*>(base), A.counters, A.out, A.epi, ctx.wd.word);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  A.smem_prefix = p.batch <= G::kPrefixCap ? 1 : 0;
  const size_t smem = G::kSmem + (A.smem_prefix ? (static_cast<size_t>(p.batch) + 1) * 4 : 0);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           G::kSmem + (G::kPrefixCap + 1) * 4) != cudaSuccess)
    return FA_ERR_CUDA;
  // programmatic dependent launch: the decode kernel starts while the plan
  // kernel runs and waits for it only before touching the counters
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_workers / kWarps));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tmk, tmv, tmk32, tmv32, A));
}

// the most workers any variant runs (int8 and bf16 at d = 64: two CTAs per
// SM); the workspace is sized for this many
int default_workers() { return min(kMaxWorkers, device_sm_count() * kMaxCtasPerSm * kWarps); }
template <int D, bool kBF>
int variant_workers() { return min(kMaxWorkers, device_sm_count() * Geom<D, kBF>::kCtas * kWarps); }

int min_tiles_of(int split_keys) { return split_keys > 0 ? split_keys / kTile : 0; }

}  // namespace

size_t decode_workspace_bytes(int batch, int hq, int head_dim) {
  // hkv is not known here: bound the group by min(hq, 8) (the kernel's
  // limit), which covers every (hkv, group) split of hq
  const size_t g = static_cast<size_t>(hq < 8 ? hq : 8);
  const size_t workers = static_cast<size_t>(default_workers());
  return plan_bytes(batch, hq) +
         (static_cast<size_t>(batch) * hq + workers * g) * (static_cast<size_t>(head_dim) + 2) * sizeof(float);
}

fa_status launch_decode(const fa_decode_params& p, const fa_kv_pages* pages, int split_keys, const LaunchCtx& ctx) {
  const int mt = min_tiles_of(split_keys);
  if (p.kv_dtype == FA_I8) {
    if (p.head_dim == 128) return launch_sk<128, false>(p, pages, variant_workers<128, false>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 64) return launch_sk<64, false>(p, pages, variant_workers<64, false>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 32) return launch_sk<32, false>(p, pages, variant_workers<32, false>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 96) return launch_sk<96, false>(p, pages, variant_workers<96, false>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 256) return launch_sk<256, false>(p, pages, variant_workers<256, false>(), mt, p.workspace, true, ctx);
  } else if (p.kv_dtype == FA_BF16) {
    if (p.head_dim == 128) return launch_sk<128, true>(p, pages, variant_workers<128, true>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 64) return launch_sk<64, true>(p, pages, variant_workers<64, true>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 32) return launch_sk<32, true>(p, pages, variant_workers<32, true>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 96) return launch_sk<96, true>(p, pages, variant_workers<96, true>(), mt, p.workspace, true, ctx);
    if (p.head_dim == 256) return launch_sk<256, true>(p, pages, variant_workers<256, true>(), mt, p.workspace, true, ctx);
  }
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
// the plan and the per-worker partials (O, m, l) live in this file-scope
// device array instead of a caller workspace.  Every device that loads the
// library holds it until the process exits.  All calls on a device share it
// and it keeps the last call's contents; nothing in it needs clearing,
// because each call writes its plan first and the merge only reads records
// that the same call's workers wrote.  Calls whose work overlaps on the GPU
// (different streams, or different host threads on the same device) race on
// the array and must be serialised by the caller.

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[kNoAllocScratchBytes];
// Status word of this path (the library's shared status word is allocated
// lazily, which this path must not do): a bounded wait that gave up, or a
// cache length outside [0, capacity].  fa_check_device_error reads and
// clears it.
static __device__ unsigned int g_decode_noalloc_status;

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};
void* g_noalloc_word[64] = {};

// Device addresses of the scratch array and status word for the current
// device.  The first call on each device looks them up (cudaGetSymbolAddress,
// with that device current); later calls reuse them.
fa_status noalloc_scratch(void** scratch, unsigned int** status) {
  void** addr = g_noalloc_addr;
  void** word = g_noalloc_word;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
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

}  // namespace

size_t decode_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Status bits the no-alloc decode recorded on the current device since the
// last read, cleared as they are read (0 before its first call there).  The
// caller has synchronised the stream; the copies are plain synchronous
// cudaMemcpy calls, which allocate nothing.
fa_status take_noalloc_status(unsigned int* bits) {
  *bits = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FA_OK;
  unsigned int* word = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    word = static_cast<unsigned int*>(g_noalloc_word[dev]);
  }
  if (word == nullptr) return FA_OK;
  if (cudaMemcpy(bits, word, sizeof(*bits), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (*bits != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Workers that fit the scratch: plan + (B*hkv + P) * G * (d + 2) floats;
// 0 when not even one CTA of workers fits.
int decode_noalloc_workers(int batch, int hq, int hkv, int head_dim) {
  const size_t fixed = plan_bytes(batch, hq) + records_bytes(batch, hq, hkv, head_dim, 0);
  if (fixed >= kNoAllocScratchBytes) return 0;
  const size_t per_worker = static_cast<size_t>(hq / hkv) * (head_dim + 2) * sizeof(float);
  const size_t fit = (kNoAllocScratchBytes - fixed) / per_worker;
  int w = static_cast<int>(fit < static_cast<size_t>(kMaxWorkers) ? fit : kMaxWorkers);
  w = min(w, default_workers());
  return (w / kWarps) * kWarps;
}

fa_status launch_decode_noalloc(const fa_decode_params& p, int split_keys, long long budget, cudaStream_t stream) {
  if (p.kv_dtype != FA_I8) return FA_ERR_UNSUPPORTED;
  const int workers = decode_noalloc_workers(p.batch, p.hq, p.hkv, p.head_dim);
  if (workers < kWarps) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  LaunchCtx ctx;
  ctx.stream = stream;
  ctx.wd.budget = budget;
  fa_status st = noalloc_scratch(&scratch, &ctx.wd.word);
  if (st != FA_OK) return st;
  // (no note_variant here: its bookkeeping set may allocate host memory)
  if (p.head_dim == 128) return launch_sk<128, false>(p, nullptr, workers, min_tiles_of(split_keys), scratch, false, ctx);
  if (p.head_dim == 64) return launch_sk<64, false>(p, nullptr, workers, min_tiles_of(split_keys), scratch, false, ctx);
  if (p.head_dim == 32) return launch_sk<32, false>(p, nullptr, workers, min_tiles_of(split_keys), scratch, false, ctx);
  if (p.head_dim == 96) return launch_sk<96, false>(p, nullptr, workers, min_tiles_of(split_keys), scratch, false, ctx);
  if (p.head_dim == 256) return launch_sk<256, false>(p, nullptr, workers, min_tiles_of(split_keys), scratch, false, ctx);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
