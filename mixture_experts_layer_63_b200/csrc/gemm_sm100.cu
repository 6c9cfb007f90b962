// Grouped GEMM on the 5th-generation tensor cores (sm_100a): TMA-fed,
// tcgen05.mma with fp32 accumulators in TMEM, fused epilogues.
//
// Serves three contractions of the layer:
//   * the bf16 router  l = x . W_r^T (+ b)         one group, fp32 out
//   * the expert up-projection, per expert segment of x_perm (and x for the
//     shared experts): ReLU(x W_i^T) (GShard section 3 of "MoE技术演进") or
//     SiLU(x W_1^T) * (x W_3^T) (SwiGLU, 3*d_model*d_moe parameters per
//     "大语言模型并行策略（七）：专家并行"), bf16 out
//   * the down-projection with the gate G_{t,e} of the combine equation
//     y_s = sum_e G_{s,e} FFN_e(x_s) folded into its epilogue, fp32 out (the
//     combine sums the rows of a token and rounds once).
// The "IO-aware" expert kernels of the Multi-Head LatentMoE summary batch
// token-to-expert traffic with the expert compute; here the batching is the
// expert-contiguous row layout and the activation / gate scaling never make
// a round trip through HBM.
//
// Kernel structure (one CTA per SM, persistent, 256 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 (bf16,
//               128-byte swizzle) per k-block into a 4-stage smem ring
//   warp 1      MMA issuer: 4 x tcgen05.mma (M=128, N=BN, K=16) per k-block,
//               tcgen05.commit frees the smem stage; a second commit hands
//               a finished accumulator to the epilogue
//   warp 2      TMEM allocation (512 columns = two 256-column accumulators)
//   warps 4-7   epilogue: tcgen05.ld of its 32 rows, activation / gate /
//               bias, bf16 pack; bf16 rows leave through a per-warp shared
//               staging buffer as whole 128-byte lines (rows beyond the
//               expert's segment are never written)
// Tiles are ordered group by group, N-tile outer and M-tile inner, so CTAs
// working at the same time share one expert's weight slice in L2.  Segment
// sizes are read from device memory inside the kernel: no host sync.
// Every wait is bounded; on expiry the kernel sets the timeout bit of the
// error word, drains its own copies and MMAs (bounded), frees TMEM and
// returns.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128;             // rows per tile (MMA M)
constexpr int BK = 64;              // bf16 elements per 128-byte swizzled row
constexpr int kUmmaK = 16;          // K per tcgen05.mma kind::f16
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr int kAccCols = 256;       // TMEM columns per accumulator buffer
constexpr int kTmemCols = 512;
constexpr int kMaxGroups = 320;
#ifndef MOE_PAIR_MIN_ROWS
#define MOE_PAIR_MIN_ROWS 384
#endif
// CTA pairs: stages of two 64-wide k-blocks where K is a multiple of 128
#ifndef MOE_PAIR_BK128
#define MOE_PAIR_BK128 1
#endif
// K-grouped weight gradients on CTA pairs as well
#ifndef MOE_PAIR_WGRAD
#define MOE_PAIR_WGRAD 1
#endif
constexpr uint32_t kABytes = BM * BK * 2;   // 16 KB
// Gathered A rows: warps 2 and 3 copy them with cp.async (16 bytes a copy,
// 128-byte swizzle applied by hand) and report a stage full after issuing
// this many later stages.  Deadlock-free for any lag below the ring depth;
// the MMA then has (depth - 1 - lag) stages ready ahead of it, so the lag is
// kept short: a lag of depth - 1 would tie every report to the completion of
// the previous stage's MMAs.
constexpr int kGatherThreads = 64;
#ifndef MOE_GATHER_LAG_ONE
#define MOE_GATHER_LAG_ONE 1
#endif
#ifndef MOE_GATHER_LAG_PAIR
#define MOE_GATHER_LAG_PAIR 2
#endif
// Stream-K tail: a piece of a split tile covers at least this many k-blocks
constexpr int kSkMinUnits = 8;
#ifndef MOE_STREAM_K
#define MOE_STREAM_K 1
#endif

struct Params {
  int epi;
  int K, N;
  int bn;           // MMA N (B tile rows)
  int bnh;          // output columns per tile (128 for SwiGLU, bn otherwise)
  int nt;           // N-tiles per group
  int n_routed, n_static, G;
  int64_t rows_static, a_static_base, a_static_stride, out_static_base;
  int64_t a_rows;
  int64_t seg_rows;         // routed segments lie in rows [0, seg_rows) (of A, or of gather_rows)
  int reverse;              // visit the tiles last group first
  const int32_t *offsets;
  void *out;
  const float *row_gate;
  const float *bias;
  int ksplit;               // K split into this many parts (router only), partial outputs
  int64_t split_stride;     //   ksplit parts of the output, split_stride elements apart
  float *sk_part;           // stream-K partial accumulators, one kSkSlotFloats slot per CTA
  int *sk_flags;            //   and one ready flag per slot; null: no stream-K
  const int32_t *gather_rows;  // routed A row r = gather_src[gather_rows[r]] (null: A as stored)
  const void *gather_src;      //   bf16 [src_rows, K]
  int64_t src_rows;
  const void *aux;          // kEpiDAct*: bf16 pre-activations [row][aux_ld]
  int64_t aux_ld;
  float *dg_part;           // kEpiDAct*: per routed row and N-tile, sum of acc * act(a)
  int dg_nt;
  const void *aux2;         // kEpiDActSwiglu: the forward's h [row][aux2_ld] for dg_part
  int64_t aux2_ld;
  const int32_t *add_rows;  // kEpiScaleAdd: output row (token) of each routed row
  int b_mn;                 // B stored [K][N] (N contiguous) instead of [N][K]
  int b_kb_split;           //   k-blocks read from map_b, the rest from map_b3
  int64_t b_krows;          //   K rows per group in B's row dimension
  int kgroup;               // K-grouped mode (weight gradients), see GroupedGemm
  int M;
  const int32_t *kseg;
  int split_m;
  int tma_store;            // token-N: whole boxes of output rows leave by TMA stores
  void *out2;
  uint32_t *err;
};

// B tiles of 128 gate rows (map_b) + 128 up rows (map_b3): SwiGLU and its
// pre-activation recompute
__host__ __device__ constexpr bool swiglu_b(int epi) {
  return epi == kEpiSwiglu || epi == kEpiPreSwiglu;
}

// Gather role: the A rows of routed tiles, one stage at a time.  Thread
// gt = 32 w + l of kGatherThreads copies 16-byte chunk c = l mod 8 of the 16
// tile rows r_i = 8 i + 4 w + l / 8: each warp-wide copy covers four whole
// 128-byte rows (coalesced).  Chunk c of row r lands at
// r * 128 + ((c ^ (r mod 8)) << 4), the 128-byte swizzle TMA would apply;
// r mod 8 is the same for all 16 rows of a thread.  Rows past the segment
// are zero-filled.
struct GatherRows {
  int32_t tok[16];             // source row of each of the thread's rows (-1: zero fill)

  __device__ __forceinline__ void load(const Params &P, int seg_off, int seg_rows, int row0, int gt) {
    const int rb = 4 * (gt >> 5) + ((gt & 31) >> 3);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = row0 + 8 * i + rb;
      int t = -1;
      if (r < seg_rows) {
        t = P.gather_rows[seg_off + r];
        if (t < 0 || t >= P.src_rows) {
          raise_error(P.err, kErrBadIndex);
          t = -1;
        }
      }
      tok[i] = t;
    }
  }
  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int i = 0; i < 16; ++i) tok[i] = -1;
  }
  __device__ __forceinline__ void issue(uint32_t sa, int gt, int kb, const char *xs,
                                        int64_t row_bytes) const {
    const int c = gt & 7;
    const int rb = 4 * (gt >> 5) + ((gt & 31) >> 3);
    const uint32_t dst0 = sa + (uint32_t)rb * 128u + ((uint32_t)(c ^ rb) << 4);
    const int64_t col = (int64_t)kb * 128 + c * 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const bool ok = tok[i] >= 0;
      cp_async_16(dst0 + (uint32_t)i * 1024u, ok ? xs + (int64_t)tok[i] * row_bytes + col : xs,
                  ok ? 16u : 0u);
    }
  }
};

// ------------------------------- tile schedule -------------------------------
struct Tile {
  int g, m, n;
};

__device__ __forceinline__ Tile decode_tile(int tile, const int *prefix, int G, int nt) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {                      // largest g with prefix[g] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  Tile t;
  t.g = lo;
  const int local = tile - prefix[lo];
  const int mt = (prefix[lo + 1] - prefix[lo]) / nt;
  t.n = local / mt;
  t.m = local - t.n * mt;
  return t;
}

// Work of one CTA (or CTA pair): whole tiles dealt round-robin, then -- when
// the tile count is not a multiple of the worker count -- a stream-K tail.
// The last tiles (between one and two waves' worth, or all of them when
// there are fewer tiles than workers) are cut into k-block units, laid end to
// end and split evenly over the workers, so no worker idles through a last,
// partly filled wave.  A tile cut between workers is summed by the worker
// holding its first k-block (the "finalizer"; that piece is the last of its
// range), adding the partial accumulators of the later workers (each one
// the first piece of its range, so it is written without waiting on anyone)
// in worker order: the result depends only on the tile count and the grid.
struct Sched {
  int P, w, KB;
  int base;                      // tiles of one K part
  int ksplit, KBs;               // router K split: parts of KBs k-blocks (no stream-K)
  int dp_rounds, dp_limit;       // round-robin items: w + i * P < dp_limit, i < dp_rounds
  int64_t sk_units;              // k-block units of the stream-K tail
  int sk_workers;                // workers sharing the tail (pieces >= kSkMinUnits)
  int64_t my_end, u;             // this worker's tail units [u, my_end)
  int i;

  __device__ __forceinline__ void init(int total, int KB_, int P_, int w_, bool sk, int ksplit_) {
    P = P_;
    w = w_;
    KB = KB_;
    base = total;
    ksplit = ksplit_ > 1 ? ksplit_ : 1;
    KBs = (KB + ksplit - 1) / ksplit;
    sk_units = 0;
    sk_workers = 1;
    if (!sk || ksplit > 1 || total % P == 0) {
      dp_limit = total * ksplit;
      dp_rounds = (dp_limit + P - 1) / P;
    } else {
      dp_rounds = total / P - 1;
      if (dp_rounds < 0) dp_rounds = 0;
      dp_limit = dp_rounds * P;
      sk_units = (int64_t)(total - dp_limit) * KB;
      int64_t nw = sk_units / kSkMinUnits;
      if (nw < 1) nw = 1;
      sk_workers = (int)(nw < P ? nw : P);
    }
    u = start(w);
    my_end = start(w + 1);
    i = 0;
  }
  // first tail unit of worker q (the tail's end for q >= sk_workers)
  __device__ __forceinline__ int64_t start(int q) const {
    return q >= sk_workers ? sk_units : (int64_t)q * sk_units / sk_workers;
  }
  // next piece of this worker: tile, k-blocks [kb0, kb1), K part
  __device__ __forceinline__ bool next(int &tile, int &kb0, int &kb1, int &part) {
    while (i < dp_rounds) {
      const int t = w + i * P;
      ++i;
      if (t < dp_limit) {
        part = t / base;
        tile = t - part * base;
        kb0 = part * KBs;
        kb1 = min(KB, kb0 + KBs);
        return true;
      }
    }
    if (u < my_end) {
      part = 0;
      tile = dp_limit + (int)(u / KB);
      kb0 = (int)(u % KB);
      const int64_t left = my_end - u;
      kb1 = (int)(KB - kb0 < left ? KB : kb0 + left);
      u += kb1 - kb0;
      return true;
    }
    return false;
  }
  // workers [w + 1, q_end) may hold later pieces of this worker's tile
  __device__ __forceinline__ int contributors_end(int tile) const {
    const int64_t tile_end = (int64_t)(tile - dp_limit + 1) * KB;
    int q = w + 1;
    while (q < sk_workers && start(q) < tile_end) ++q;
    return q;
  }
  __device__ __forceinline__ bool nonempty(int q) const { return start(q + 1) > start(q); }
};

// Stream-K partial accumulator slot: 128 rows x 256 fp32 columns, stored as
// float4 column groups of 128 rows, so that a warp's 32 rows x 16 bytes are
// one contiguous 512-byte run.
__device__ __forceinline__ float4 *sk_slot_ptr(float *part, int slot, int row, int col) {
  return reinterpret_cast<float4 *>(part + (size_t)slot * kSkSlotFloats) + (size_t)(col >> 2) * BM + row;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add_gpu(int *p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Ready flags count rows, so no epilogue thread ever waits on another thread
// of its own CTA: each of the 128 writer threads adds 1 after storing its row
// (release); a finalizer thread reads a slot once the flag is >= 128
// (acquire) and then adds 1 itself; the thread that brings it to 256 resets
// it to 0 for the next launch, which the stream orders after this one.
constexpr int kEpiThreads = 128;

// The finalizer's view of the later pieces of its tile: slots of workers
// q in [q0, q1) with a non-empty range, slot = q * slot_mul + slot_add.
struct Fixup {
  const float *part;
  const Sched *sc;
  int q0, q1, slot_mul, slot_add, row;
};

// v[i] += every later piece's column col + i of this row, in worker order
__device__ __forceinline__ void add_parts(float (&v)[32], const Fixup &F, int col) {
  for (int q = F.q0; q < F.q1; ++q) {
    if (!F.sc->nonempty(q)) continue;
    const float4 *p = sk_slot_ptr(const_cast<float *>(F.part), q * F.slot_mul + F.slot_add, F.row, col);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 t = p[(size_t)j * BM];
      v[4 * j + 0] += t.x;
      v[4 * j + 1] += t.y;
      v[4 * j + 2] += t.z;
      v[4 * j + 3] += t.w;
    }
  }
}

// A piece that does not finish its tile: this thread's row of the raw
// accumulator (P.bn TMEM columns) into the worker's slot, then publish it.
__device__ __forceinline__ void sk_write(const Params &P, int slot, int row, uint32_t taddr) {
  uint32_t r[32];
#pragma unroll 1
  for (int c = 0; c < P.bn; c += 32) {
    tmem_ld32(taddr + c, r);
    tmem_ld_wait();
    float4 *p = sk_slot_ptr(P.sk_part, slot, row, c);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      p[(size_t)j * BM] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                      __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
  }
  red_release_add_gpu(P.sk_flags + slot, 1);
}

// Finalizer thread: bounded wait until every later piece of the tile is
// published.  False when the CTA is aborting (timeout bit raised here).
__device__ __forceinline__ bool sk_wait(const Params &P, const Fixup &F, volatile int *abort_flag,
                                        uint64_t limit) {
  for (int q = F.q0; q < F.q1; ++q) {
    if (!F.sc->nonempty(q)) continue;
    const int *flag = P.sk_flags + q * F.slot_mul + F.slot_add;
    if (ld_acquire_gpu(flag) >= kEpiThreads) continue;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ld_acquire_gpu(flag) >= kEpiThreads) break;
      if ((it & 63u) == 0) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit) {
          raise_error(P.err, kErrTimeout);
          *abort_flag = 1;
          return false;
        }
      }
    }
  }
  return true;
}

// Finalizer thread, after its epilogue read the slots: count itself done;
// the last of the 128 readers clears the flag.
__device__ __forceinline__ void sk_done(const Params &P, const Fixup &F) {
  for (int q = F.q0; q < F.q1; ++q) {
    if (!F.sc->nonempty(q)) continue;
    int *flag = P.sk_flags + q * F.slot_mul + F.slot_add;
    if (atomicAdd(flag, 1) == 2 * kEpiThreads - 1) atomicExch(flag, 0);
  }
}

// --------------------------------- epilogues ---------------------------------
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16 *src, float (&v)[32]) {
  const uint4 *p = reinterpret_cast<const uint4 *>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = p[q];
    v[8 * q + 0] = bf16_lo(w.x); v[8 * q + 1] = bf16_hi(w.x);
    v[8 * q + 2] = bf16_lo(w.y); v[8 * q + 3] = bf16_hi(w.y);
    v[8 * q + 4] = bf16_lo(w.z); v[8 * q + 5] = bf16_hi(w.z);
    v[8 * q + 6] = bf16_lo(w.w); v[8 * q + 7] = bf16_hi(w.w);
  }
}

// bf16 outputs leave through a 4 KB staging buffer of the warp in shared
// memory: each thread writes its row's PIECES 16-byte pieces there (piece c
// of row r at slot c ^ f(r), which keeps both the writes and the reads below
// free of bank conflicts), then every store instruction of the warp writes
// 32 / PIECES whole rows of PIECES * 16 bytes (8 pieces: 128-byte lines).
// Stored straight from the row-per-thread layout, a warp's 16-byte stores
// would touch 32 rows each and fill every 32-byte sector in two halves.
// Row r of the warp (output row row0 + r) is written when bit r of vmask is
// set.
constexpr int kStageBytesPerWarp = 32 * 128;

template <int PIECES>
__device__ __forceinline__ int stage_slot(int r, int c) {
  return PIECES == 8 ? c ^ (r & 7) : c ^ ((r >> 1) & 3);
}

template <int PIECES>
__device__ __forceinline__ void store_rows(uint8_t *stg, const uint32_t (&pk)[PIECES * 4],
                                           __nv_bfloat16 *out, int64_t ld, int64_t row0, int col,
                                           uint32_t vmask, int lane) {
  static_assert(PIECES == 4 || PIECES == 8, "rows of 64 or 128 bytes");
  constexpr int kRowBytes = PIECES * 16;
  constexpr int kRowsPerStore = 32 / PIECES;
  uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * kRowBytes);
#pragma unroll
  for (int c = 0; c < PIECES; ++c)
    mine[stage_slot<PIECES>(lane, c)] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int p = 0; p < PIECES; ++p) {
    const int r = p * kRowsPerStore + lane / PIECES, c = lane % PIECES;
    const uint4 w = reinterpret_cast<const uint4 *>(stg + r * kRowBytes)[stage_slot<PIECES>(r, c)];
    if ((vmask >> r) & 1u) *reinterpret_cast<uint4 *>(out + (row0 + r) * ld + col + c * 8) = w;
  }
  __syncwarp();
}

// store_rows<8> for a warp whose 32 rows are all to be written, through
// one TMA store: the staging above already holds piece c of row r at slot
// c ^ (r mod 8), the layout of a 128-byte-swizzled box of 32 rows x 64
// columns (the staging buffer is 1024-byte aligned).  The next use of the
// staging waits until the store has read it.
__device__ __forceinline__ void store_rows_tma(uint8_t *stg, const uint32_t (&pk)[32],
                                               const CUtensorMap *omap, int64_t row0, int col,
                                               int lane) {
  uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    mine[stage_slot<8>(lane, c)] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(omap, stg, col, (int)row0);
    bulk_commit();
  }
}

// The same staging, with the rows added into out (bf16, vector reductions)
// at rows dest of each thread's row (-1: not added) instead of stored.
__device__ __forceinline__ void red_add_bf16x8(__nv_bfloat16 *p, const uint4 w) {
  asm volatile("red.global.add.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(w.x), "r"(w.y),
               "r"(w.z), "r"(w.w)
               : "memory");
}

__device__ __forceinline__ void red_rows(uint8_t *stg, const uint32_t (&pk)[32], __nv_bfloat16 *out,
                                         int64_t ld, int dest, int col, int lane) {
  uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    mine[stage_slot<8>(lane, c)] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int r = p * 4 + (lane >> 3), c = lane & 7;
    const uint4 w = reinterpret_cast<const uint4 *>(stg + r * 128)[stage_slot<8>(r, c)];
    const int dr = __shfl_sync(0xffffffffu, dest, r);
    if (dr >= 0) red_add_bf16x8(out + (int64_t)dr * ld + col + c * 8, w);
  }
  __syncwarp();
}

// Each thread's 128-byte row piece (32 words) to its own destination `dst`
// (bytes; null: not stored), through the warp's staging buffer: every store
// instruction of the warp then writes four whole 128-byte lines.
__device__ __forceinline__ void store_rows_at(uint8_t *stg, const uint32_t (&pk)[32], char *dst, int lane) {
  uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    mine[stage_slot<8>(lane, c)] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int r = p * 4 + (lane >> 3), c = lane & 7;
    const uint4 w = reinterpret_cast<const uint4 *>(stg + r * 128)[stage_slot<8>(r, c)];
    char *d = reinterpret_cast<char *>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), r));
    if (d) *reinterpret_cast<uint4 *>(d + c * 16) = w;
  }
  __syncwarp();
}

// 32 fp32 values into 16 bf16x2 words at word offset 16 * H of pk
template <int H, int N>
__device__ __forceinline__ void pack_words(uint32_t (&pk)[N], const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[16 * H + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
}

// TMEM columns [c, c + 32) of this thread's row as fp32, plus the later
// stream-K pieces of the tile when F is given
__device__ __forceinline__ void acc_cols(uint32_t taddr, int c, const Fixup *F, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr + c, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (F) add_parts(v, *F, c);
}

// Epilogue of one accumulator: this thread's row (TMEM lane) of the tile,
// BN columns from TMEM address `taddr` (SwiGLU forms: gate columns 0-127,
// up 128-255), output columns from col0 on; the later stream-K pieces of the
// tile added first when F is given; then activation / gate / bias, stores.
// The warp's rows are consecutive (lane l: output row out_row = row0 + l);
// `stg` is the warp's staging buffer.  kEpiScaleAdd adds the row into output
// row `dest` instead (-1: nothing).
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const Params &P, uint32_t taddr, bool valid, bool routed,
                                              int64_t out_row, int col0, uint8_t *stg, int lane,
                                              int64_t out_offset = 0, const Fixup *F = nullptr,
                                              int dest = -1, const CUtensorMap *omap = nullptr) {
  float v[32];
  if constexpr (EPI == kEpiStoreF32) {
    // a K part when the router is split: no bias, own output
    float *out = reinterpret_cast<float *>(P.out) + out_offset;
    const float *bias = P.ksplit > 1 ? nullptr : P.bias;
#pragma unroll 1
    for (int c = 0; c < P.bn / 32; ++c) {
      acc_cols(taddr, c * 32, F, v);
      const int col0c = col0 + c * 32;
      if (col0c >= P.N) break;                                  // the same for the whole CTA
      if (!bias && col0c + 32 <= P.N && (P.N & 3) == 0) {
        // whole 32-column groups: 128-byte rows through the staging buffer
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
        store_rows_at(stg, w, valid ? reinterpret_cast<char *>(out + out_row * P.N + col0c) : nullptr,
                      lane);
      } else if (valid) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = col0c + i;
          if (col < P.N) out[out_row * P.N + col] = bias ? v[i] + bias[col] : v[i];
        }
      }
    }
    return;
  }
  __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(P.out);
  const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
  const int64_t row0 = out_row - lane;
  if constexpr (EPI == kEpiPreSwiglu || EPI == kEpiDActSwiglu) {
    // two outputs: [row][col] and [row][N + col], 32 columns at a time
    const int64_t ld = 2 * (int64_t)P.N;
    const int ncol = EPI == kEpiPreSwiglu ? 128 : P.bn;
    const float scale = (EPI == kEpiDActSwiglu && routed && valid) ? P.row_gate[out_row] : 1.0f;
    const __nv_bfloat16 *aux = reinterpret_cast<const __nv_bfloat16 *>(P.aux);
    float dg = 0.0f;                                            // sum of acc * h (the forward's h)
#pragma unroll 1
    for (int c = 0; c < ncol / 32; ++c) {
      const int col = col0 + c * 32;
      if (col >= P.N) break;                                    // the same for the whole CTA
      float w[32];
      uint32_t pk[16], pk2[16];
      if constexpr (EPI == kEpiPreSwiglu) {
        acc_cols(taddr, c * 32, F, v);                          // a
        acc_cols(taddr, 128 + c * 32, F, w);                    // u
      } else {
        // dh = g * acc, then SwiGLU's backward from the saved a and u
        acc_cols(taddr, c * 32, F, v);
        if (P.dg_part && routed && valid) {
          // gate-gradient piece against the forward's h (rounded once)
          float hh[32];
          load_bf16x32(reinterpret_cast<const __nv_bfloat16 *>(P.aux2) + out_row * P.aux2_ld + col, hh);
#pragma unroll
          for (int i = 0; i < 32; ++i) dg = fmaf(v[i], hh[i], dg);
        }
        float a[32], uu[32];
        if (valid) {
          load_bf16x32(aux + out_row * P.aux_ld + col, a);
          load_bf16x32(aux + out_row * P.aux_ld + P.N + col, uu);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = uu[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sg = sigmoid_f(a[i]);
          const float dh = v[i] * scale;
          w[i] = dh * a[i] * sg;
          v[i] = dh * uu[i] * sg * (1.0f + a[i] * (1.0f - sg));
        }
      }
      pack_words<0>(pk, v);
      pack_words<0>(pk2, w);
      store_rows<4>(stg, pk, out, ld, row0, col, vmask, lane);
      store_rows<4>(stg, pk2, out, ld, row0, (int)P.N + col, vmask, lane);
    }
    if (EPI == kEpiDActSwiglu && P.dg_part && routed && valid)
      P.dg_part[out_row * P.dg_nt + col0 / P.bnh] = dg;
  } else {
    // one output, 64 columns (one 128-byte line a row) at a time
    const int ncol = EPI == kEpiSwiglu ? 128 : P.bn;
    const int64_t ld = P.N;
    const float scale = ((EPI == kEpiScale || EPI == kEpiScaleAdd || EPI == kEpiDActRelu) && routed && valid)
                            ? P.row_gate[out_row] : 1.0f;
    const __nv_bfloat16 *aux = reinterpret_cast<const __nv_bfloat16 *>(P.aux);
    float dg = 0.0f;                                            // sum of acc * relu(a)
#pragma unroll 1
    for (int c2 = 0; c2 < ncol / 64; ++c2) {
      const int col = col0 + c2 * 64;
      if (col >= P.N) break;                                    // the same for the whole CTA
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 2 * c2 + h;                               // 32-column group of the tile
        acc_cols(taddr, c * 32, F, v);
        if constexpr (EPI == kEpiSwiglu) {
          float uf[32];
          acc_cols(taddr, 128 + c * 32, F, uf);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu_f(v[i]) * uf[i];
        } else if constexpr (EPI == kEpiRelu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], 0.0f);
        } else if constexpr (EPI == kEpiScale || EPI == kEpiScaleAdd) {
          // gated rows in bf16; the combine sums them in fp32 and rounds once
          // (kEpiScaleAdd: added into the zeroed output rows, at most two per row)
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= scale;
        } else if constexpr (EPI == kEpiDActRelu) {
          // dh = g * acc, masked where the saved pre-activation a <= 0
          float a[32];
          if (valid) {
            load_bf16x32(aux + out_row * P.aux_ld + col + h * 32, a);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = 0.f;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            dg = fmaf(v[i], fmaxf(a[i], 0.0f), dg);
            v[i] = a[i] > 0.0f ? v[i] * scale : 0.0f;
          }
        }                                                       // kEpiPreRelu: a as is
        if (h == 0) pack_words<0>(pk, v);
        else pack_words<1>(pk, v);
      }
      if (P.tma_store) {                                       // the last TMA store has read stg
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      if constexpr (EPI == kEpiScaleAdd) red_rows(stg, pk, out, ld, dest, col, lane);
      else if (P.tma_store && omap && vmask == 0xffffffffu) store_rows_tma(stg, pk, omap, row0, col, lane);
      else store_rows<8>(stg, pk, out, ld, row0, col, vmask, lane);
    }
    if (EPI == kEpiDActRelu && P.dg_part && routed && valid)
      P.dg_part[out_row * P.dg_nt + col0 / P.bnh] = dg;
  }
}

// kEpiScaleAdd: the output row a tile row adds into (its token; a static
// group's row t is token t), -1 when out of range (error bit raised)
__device__ __forceinline__ int add_dest(const Params &P, bool routed, int64_t out_row, int64_t tile_row) {
  const int64_t t = routed ? (int64_t)P.add_rows[out_row] : tile_row;
  if (t < 0 || t >= P.src_rows) {
    raise_error(P.err, kErrBadIndex);
    return -1;
  }
  return (int)t;
}

// K-grouped mode: this thread's row of a weight-gradient tile (fp32), or
// zeros when the group has no K columns (zero is the same for the whole
// CTA, so the warp's TMEM loads stay aligned); dst null: row past M.  Whole
// 32-column groups (128 bytes a row) leave through the staging buffer.
// `om`: the fp32 tensor map of the output part that holds all 32 rows of
// this warp, `orow` the first of them there; whole 32-row x 32-column pieces
// then leave by TMA stores from the 128-byte-swizzled staging (the pieces
// of the last columns by plain stores).  Null: plain stores throughout.
__device__ __forceinline__ void epilogue_wgrad(const Params &P, uint32_t taddr, bool zero, float *dst,
                                               int col0, uint8_t *stg, int lane,
                                               const CUtensorMap *om = nullptr, int64_t orow = 0) {
  uint32_t r[32];
#pragma unroll 1
  for (int c = 0; c < P.bn / 32; ++c) {
    const int col = col0 + c * 32;
    if (!zero) {
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    if (col >= P.N) break;                                      // the same for the whole CTA
    if (P.tma_store) {                                          // the last TMA store has read stg
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
    }
    if (om && col + 32 <= P.N) {
      uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * 128);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        mine[stage_slot<8>(lane, q)] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(om, stg, col, (int)orow);
        bulk_commit();
      }
    } else if (col + 32 <= P.N && (P.N & 3) == 0) {
      store_rows_at(stg, r, dst ? reinterpret_cast<char *>(dst + col) : nullptr, lane);
    } else if (dst) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col + i < P.N) dst[col + i] = __uint_as_float(r[i]);
    }
  }
}

// --------------------------------- the kernel --------------------------------
template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_a_static,
                        const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_b3,
                        const __grid_constant__ CUtensorMap map_out, const Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int s_prefix[kMaxGroups + 1];
  __shared__ int s_off[kMaxGroups];
  __shared__ int s_rows[kMaxGroups];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ uint64_t s_limit_sh;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t b_bytes = (uint32_t)P.bn * BK * 2;
  const uint32_t stage_bytes = kABytes + b_bytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const bool gather = P.gather_rows != nullptr;
  if (tid == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1 + (gather ? kGatherThreads / 32 : 0));   // + one per gather warp
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf_bar[a], 1);
      mbar_init(&acce_bar[a], 4 * 32);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    tma_prefetch_map(&map_a);
    tma_prefetch_map(&map_b);
    if (P.n_static > 0) tma_prefetch_map(&map_a_static);
    if (swiglu_b(EPI)) tma_prefetch_map(&map_b3);
  }
  pdl_wait();              // what earlier kernels wrote is visible from here on
  pdl_trigger();
  if (tid == 0) s_limit_sh = wait_limit_ns(P.err);
  // group table: rows and tile prefix, warp 0
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < P.G; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < P.G && P.kgroup) {
        // K-grouped: group g owns K columns [kseg[g], kseg[g+1]); rows = its k-blocks
        const int k0 = P.kseg[g], k1 = P.kseg[g + 1];
        const int kbg = (k1 - k0) / BK;
        if (k0 < 0 || k1 < k0 || (k0 % BK) != 0 || (int64_t)k1 > P.a_rows) {
          raise_error(P.err, kErrBadIndex);
          s_off[g] = 0;
          s_rows[g] = 0;
        } else {
          s_off[g] = k0;
          s_rows[g] = kbg;
        }
        tiles = ((P.M + BM - 1) / BM) * P.nt;
      } else if (g < P.G) {
        int off = 0, rows = 0;
        if (g < P.n_routed) {
          off = P.offsets[g];
          rows = P.offsets[g + 1] - off;
          if (rows < 0 || off < 0 || (int64_t)off + rows > P.seg_rows) {
            raise_error(P.err, kErrBadIndex);
            rows = 0;
            off = 0;
          }
        } else {
          rows = (int)P.rows_static;
        }
        s_off[g] = off;
        s_rows[g] = rows;
        tiles = ((rows + BM - 1) / BM) * P.nt;
      }
      int x = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (g < P.G) s_prefix[g] = carry + x - tiles;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_prefix[P.G] = carry;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const uint64_t s_limit = s_limit_sh;
  const int KB = P.K / BK;
  const bool sk = EPI != kEpiStoreF32 && P.sk_part != nullptr;
  Sched sc;
  sc.init(s_prefix[P.G], KB, gridDim.x, blockIdx.x, sk, P.ksplit);
  int tile, kb0, kb1, part;

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0;            // bit s: full_bar[s] armed and maybe in flight
    uint32_t armed_parity = 0;     // bit s: parity of that phase
    bool ok = true;
    // operand coordinates of a tile
    auto a_of = [&](const Tile &tl, int64_t &row) -> const CUtensorMap * {
      const bool routed = tl.g < P.n_routed;
      row = routed ? (int64_t)s_off[tl.g] + (int64_t)tl.m * BM
                   : P.a_static_base + (int64_t)(tl.g - P.n_routed) * P.a_static_stride +
                         (int64_t)tl.m * BM;
      return routed ? &map_a : &map_a_static;
    };
    while (ok && sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      int64_t a_row;
      const CUtensorMap *ma = a_of(tl, a_row);
      int b_row = tl.g * P.N + tl.n * P.bnh;
      int kx = 0;                      // K coordinate of k-block 0
      if (P.kgroup) {
        ma = &map_a;
        a_row = (int64_t)tl.m * BM;
        b_row = tl.n * P.bnh;
        kx = s_off[tl.g];
        kb0 = 0;
        kb1 = s_rows[tl.g];
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
        uint8_t *sa = smem + (size_t)stage * stage_bytes;
        uint8_t *sb = sa + kABytes;
        const bool a_by_tma = !(gather && tl.g < P.n_routed);   // else the gather warps
        mbar_expect_tx(&full_bar[stage], a_by_tma ? stage_bytes : b_bytes);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (a_by_tma) tma_load_2d(sa, ma, &full_bar[stage], kx + kb * BK, (int)a_row);
        if (P.b_mn) {
          // B as [K][N]: bn/64 boxes of 64 N x 64 K, 8 KB apart
          const bool first = kb < P.b_kb_split;
          const int y = (int)(tl.g * P.b_krows) + (first ? kb : kb - P.b_kb_split) * BK;
          for (int j = 0; j < P.bn / 64; ++j)
            tma_load_2d(sb + j * 8192, first ? &map_b : &map_b3, &full_bar[stage],
                        tl.n * P.bnh + j * 64, y);
        } else if (swiglu_b(EPI)) {
          tma_load_2d(sb, &map_b, &full_bar[stage], kx + kb * BK, b_row);
          tma_load_2d(sb + (b_bytes >> 1), &map_b3, &full_bar[stage], kx + kb * BK, b_row);
        } else {
          tma_load_2d(sb, &map_b, &full_bar[stage], kx + kb * BK, b_row);
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {
      // aborting: let the copies already issued land before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if (armed & (1u << s)) mbar_wait_drain(&full_bar[s], (armed_parity >> s) & 1u);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------- MMA issuer -------------------------------
    const uint32_t idesc = idesc_bf16(BM, P.bn) | (P.b_mn ? (1u << 16) : 0u);   // bit 16: B MN-major
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    while (ok && sc.next(tile, kb0, kb1, part)) {
      if (P.kgroup) {
        const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
        kb0 = 0;
        kb1 = s_rows[tl.g];
      }
      if (!mbar_wait(&acce_bar[acc], acc_phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, &s_abort, P.err, s_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + (size_t)stage * stage_bytes);
        const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
        for (int k = 0; k < BK / kUmmaK; ++k) {
          const uint64_t bdesc = P.b_mn ? mn128_desc(b_addr + k * 2048) : sw128_desc(b_addr + k * kUmmaK * 2);
          umma_bf16(d_tmem, sw128_desc(a_addr + k * kUmmaK * 2), bdesc, idesc,
                    (kb > kb0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit(&accf_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // all MMAs issued by this thread complete before TMEM can be freed
    umma_commit(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  } else if (gather && (warp == 2 || warp == 3)) {
    // ------------------------- gather of routed A rows -------------------------
    constexpr int kLag = MOE_GATHER_LAG_ONE;
    static_assert(kLag >= 0 && kLag < kStages, "gather lag below the ring depth");
    const int gt = tid - 64;
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0, arrived = 0;
    bool ok = true;
    const char *xs = static_cast<const char *>(P.gather_src);
    const int64_t row_bytes = (int64_t)P.K * 2;
    while (ok && sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      const bool routed = tl.g < P.n_routed;
      GatherRows gr;
      if (routed) gr.load(P, s_off[tl.g], s_rows[tl.g], tl.m * BM, gt);
      else gr.clear();
      for (int kb = kb0; kb < kb1; ++kb) {
        // lane 0 waits for the stage to be free, the warp follows it
        int okw = 1;
        if (lane == 0) okw = mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, s_limit) ? 1 : 0;
        __syncwarp();
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        if (routed) gr.issue(smem_u32(smem + (size_t)stage * stage_bytes), gt, kb, xs, row_bytes);
        cp_async_commit();
        ++issued;
        if (issued - arrived > kLag) {
          cp_async_wait<kLag>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full_bar[arrived % kStages]);   // one arrival per warp
          ++arrived;
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    for (; arrived < issued; ++arrived)
      if (lane == 0) mbar_arrive(&full_bar[arrived % kStages]);
  } else if (warp >= 4) {
    // -------------------------------- epilogue --------------------------------
    const int ew = warp - 4;                     // TMEM lanes 32*ew .. 32*ew+31
    const int r_cta = ew * 32 + lane;            // row of the tile
    uint8_t *stg = smem + (size_t)kStages * stage_bytes + (size_t)ew * kStageBytesPerWarp;
    int acc = 0;
    uint32_t acc_phase = 0;
    while (sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      // (warp-uniform exits: the epilogue's TMEM loads and stores are warp-wide)
      if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[acc], acc_phase, &s_abort, P.err, s_limit))) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * kAccCols) + ((uint32_t)(ew * 32) << 16);
      const bool in_tail = sk && tile >= sc.dp_limit;
      if (P.kgroup) {
        // weight gradient tile: rows of group g's [M, N] output (split at split_m)
        const int row = tl.m * BM + r_cta;
        const bool zero = s_rows[tl.g] == 0;
        float *dst = nullptr;
        if (row < P.M)
          dst = row < P.split_m
                    ? reinterpret_cast<float *>(P.out) + ((int64_t)tl.g * P.split_m + row) * P.N
                    : reinterpret_cast<float *>(P.out2) +
                          ((int64_t)tl.g * (P.M - P.split_m) + row - P.split_m) * P.N;
        epilogue_wgrad(P, taddr, zero, dst, tl.n * P.bnh, stg, lane);
      } else if (in_tail && kb0 > 0) {
        sk_write(P, (int)blockIdx.x, r_cta, taddr);              // a later piece of the tile
      } else {
        const bool routed = tl.g < P.n_routed;
        const bool valid = tl.m * BM + r_cta < s_rows[tl.g];
        const int64_t out_row = (routed ? (int64_t)s_off[tl.g]
                                        : P.out_static_base + (int64_t)(tl.g - P.n_routed) * P.rows_static) +
                                (int64_t)tl.m * BM + r_cta;
        const int col0 = tl.n * P.bnh;
        const int dest = (EPI == kEpiScaleAdd && valid) ? add_dest(P, routed, out_row, tl.m * BM + r_cta) : -1;
        if (in_tail && kb1 < KB) {                              // finalizer of a split tile
          const Fixup F{P.sk_part, &sc, (int)blockIdx.x + 1, sc.contributors_end(tile), 1, 0, r_cta};
          if (!__all_sync(0xffffffffu, sk_wait(P, F, &s_abort, s_limit))) break;
          epilogue_tile<EPI>(P, taddr, valid, routed, out_row, col0, stg, lane, 0, &F, dest, &map_out);
          sk_done(P, F);
        } else {
          epilogue_tile<EPI>(P, taddr, valid, routed, out_row, col0, stg, lane,
                             (int64_t)part * P.split_stride, nullptr, dest, &map_out);
        }
      }
      tc_fence_before();
      mbar_arrive(&acce_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (P.tma_store && lane == 0) bulk_wait_all();     // this warp's TMA stores written
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}


// ------------------------- the kernel, CTA-pair version -----------------------
// Same contract as grouped_gemm_kernel, tiles of 256 rows: the two CTAs of a
// cluster each stage 128 rows of A and half of the B tile (BN/2 rows) per
// k-block, and the even CTA issues tcgen05.mma.cta_group::2 (M = 256), which
// reads both CTAs' shared memory and leaves rows 0-127 of the accumulator in
// the even CTA's TMEM and rows 128-255 in the odd CTA's.  Each CTA moves 32 KB
// per k-block instead of 48 KB for the same MMA work.  Both CTAs' TMA loads
// complete on the even CTA's full barrier; the MMA commits arrive on the
// empty / accumulator-full barriers of both CTAs; both CTAs' epilogues arrive
// on the even CTA's accumulator-empty barrier.  No load is multicast.
//
// BKS = 2: stages of two 64-wide k-blocks (three 64 KB stages instead of six
// of 32 KB, eight MMAs and one barrier round trip per stage), for K a
// multiple of 128 without the row gather, K-major B only.
constexpr int kPairStages = 6;
constexpr int kPairStages2 = 3;

template <int EPI, int BKS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                             const __grid_constant__ CUtensorMap map_a_static,
                             const __grid_constant__ CUtensorMap map_b,
                             const __grid_constant__ CUtensorMap map_b3,
                             const __grid_constant__ CUtensorMap map_out,
                             const __grid_constant__ CUtensorMap map_out2, const Params P) {
  constexpr int PM = 2 * BM;                         // rows per pair tile
  constexpr int STAGES = BKS == 2 ? kPairStages2 : kPairStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int s_prefix[kMaxGroups + 1];
  __shared__ int s_off[kMaxGroups];
  __shared__ int s_rows[kMaxGroups];
  __shared__ __align__(8) uint64_t full_bar[kPairStages];
  __shared__ __align__(8) uint64_t empty_bar[kPairStages];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ uint64_t s_limit_sh;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t b_bytes = (uint32_t)(P.bn / 2) * BK * 2;       // this CTA's half of B
  const uint32_t stage_bytes = BKS * (kABytes + b_bytes);       // A blocks, then B blocks
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const bool gather = P.gather_rows != nullptr;
  if (tid == 32) {
    for (int st = 0; st < STAGES; ++st) {
      // the even CTA's: its expect_tx arrival, then both CTAs' gather warps
      mbar_init(&full_bar[st], 1 + (gather ? 2 * kGatherThreads / 32 : 0));
      mbar_init(&empty_bar[st], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf_bar[a], 1);
      mbar_init(&acce_bar[a], 2 * 4 * 32);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  if (tid == 0) {
    tma_prefetch_map(&map_a);
    tma_prefetch_map(&map_b);
    if (P.n_static > 0) tma_prefetch_map(&map_a_static);
    if (swiglu_b(EPI)) tma_prefetch_map(&map_b3);
  }
  pdl_wait();              // what earlier kernels wrote is visible from here on
  pdl_trigger();
  if (tid == 0) s_limit_sh = wait_limit_ns(P.err);
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < P.G; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < P.G && P.kgroup) {
        // K-grouped: group g owns K columns [kseg[g], kseg[g+1]); rows = its k-blocks
        const int k0 = P.kseg[g], k1 = P.kseg[g + 1];
        if (k0 < 0 || k1 < k0 || (k0 % BK) != 0 || (int64_t)k1 > P.a_rows) {
          raise_error(P.err, kErrBadIndex);
          s_off[g] = 0;
          s_rows[g] = 0;
        } else {
          s_off[g] = k0;
          s_rows[g] = (k1 - k0) / BK;
        }
        tiles = ((P.M + PM - 1) / PM) * P.nt;
      } else if (g < P.G) {
        int off = 0, rows = 0;
        if (g < P.n_routed) {
          off = P.offsets[g];
          rows = P.offsets[g + 1] - off;
          if (rows < 0 || off < 0 || (int64_t)off + rows > P.seg_rows) {
            raise_error(P.err, kErrBadIndex);
            rows = 0;
            off = 0;
          }
        } else {
          rows = (int)P.rows_static;
        }
        s_off[g] = off;
        s_rows[g] = rows;
        tiles = ((rows + PM - 1) / PM) * P.nt;
      }
      int x = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (g < P.G) s_prefix[g] = carry + x - tiles;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_prefix[P.G] = carry;
  }
  tc_fence_before();
  cluster_sync_all();              // barriers of both CTAs initialised before any remote use
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const uint64_t s_limit = s_limit_sh;
  const int KB = P.K / (BK * BKS);                     // stages of K per tile
  const bool sk = P.sk_part != nullptr;
  Sched sc;
  sc.init(s_prefix[P.G], KB, npairs, pair, sk, 1);
  int tile, kb0, kb1, part;

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    // B rows of this CTA: SwiGLU: even CTA the gate rows (W1), odd CTA the up
    // rows (W3); otherwise the two halves of the BN-row tile
    const CUtensorMap *mb = (swiglu_b(EPI) && rank == 1) ? &map_b3 : &map_b;
    auto rows_of = [&](const Tile &tl, int64_t &a_row, int &b_row) -> const CUtensorMap * {
      const bool routed = tl.g < P.n_routed;
      a_row = (routed ? (int64_t)s_off[tl.g]
                      : P.a_static_base + (int64_t)(tl.g - P.n_routed) * P.a_static_stride) +
              (int64_t)tl.m * PM + (int64_t)rank * BM;
      b_row = tl.g * P.N + tl.n * P.bnh + (swiglu_b(EPI) ? 0 : (int)rank * (P.bn / 2));
      return routed ? &map_a : &map_a_static;
    };
    while (ok && sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      int64_t a_row;
      int b_row;
      const CUtensorMap *ma = rows_of(tl, a_row, b_row);
      int kx = 0;                      // K coordinate of k-block 0
      if (P.kgroup) {
        // weight gradient: A [M, K] rows of this CTA, B [N, K] half of the tile
        ma = &map_a;
        a_row = (int64_t)tl.m * PM + (int64_t)rank * BM;
        b_row = tl.n * P.bnh + (int)rank * (P.bn / 2);
        kx = s_off[tl.g];
        kb0 = 0;
        kb1 = s_rows[tl.g];
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
        uint8_t *sa = smem + (size_t)stage * stage_bytes;
        uint8_t *sb = sa + BKS * kABytes;
        const uint32_t fb = smem_u32(&full_bar[stage]) & 0xFEFFFFFFu;   // the even CTA's barrier
        const bool a_by_tma = !(gather && tl.g < P.n_routed);          // else the gather warps
        if (rank == 0) {
          mbar_expect_tx(&full_bar[stage], a_by_tma ? 2 * stage_bytes : 2 * b_bytes);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        if (a_by_tma) {
#pragma unroll
          for (int q = 0; q < BKS; ++q)
            tma_load_2d_pair(sa + q * kABytes, ma, fb, kx + (kb * BKS + q) * BK, (int)a_row);
        }
        if (P.b_mn) {
          // this CTA's 128 N columns of B stored [K][N]: two boxes of 64 N x 64 K
          const bool first = kb < P.b_kb_split;
          const int y = (int)(tl.g * P.b_krows) + (first ? kb : kb - P.b_kb_split) * BK;
          for (int j = 0; j < P.bn / 128; ++j)
            tma_load_2d_pair(sb + j * 8192, first ? &map_b : &map_b3, fb,
                             tl.n * P.bnh + (int)rank * (P.bn / 2) + j * 64, y);
        } else {
#pragma unroll
          for (int q = 0; q < BKS; ++q)
            tma_load_2d_pair(sb + q * b_bytes, mb, fb, kx + (kb * BKS + q) * BK, b_row);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && rank == 0) {
      for (int st = 0; st < STAGES; ++st)
        if (armed & (1u << st)) mbar_wait_drain(&full_bar[st], (armed_parity >> st) & 1u);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------ MMA issuer (even CTA only) ------------------------
    const uint32_t idesc = idesc_bf16(PM, P.bn) | (P.b_mn ? (1u << 16) : 0u);   // bit 16: B MN-major
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    while (ok && sc.next(tile, kb0, kb1, part)) {
      if (P.kgroup) {
        const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
        kb0 = 0;
        kb1 = s_rows[tl.g];
      }
      if (!mbar_wait(&acce_bar[acc], acc_phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait<true>(&full_bar[stage], phase, &s_abort, P.err, s_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + (size_t)stage * stage_bytes);
        const uint32_t b_addr = a_addr + BKS * kABytes;
#pragma unroll
        for (int q = 0; q < BKS; ++q) {
#pragma unroll
          for (int k = 0; k < BK / kUmmaK; ++k) {
            const uint32_t bq = b_addr + q * b_bytes;
            const uint64_t bdesc = P.b_mn ? mn128_desc(bq + k * 2048) : sw128_desc(bq + k * kUmmaK * 2);
            umma_bf16_pair(d_tmem, sw128_desc(a_addr + q * kABytes + k * kUmmaK * 2), bdesc, idesc,
                           (kb > kb0 || q > 0 || k > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair_both(&empty_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit_pair_both(&accf_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    umma_commit_pair_local(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  } else if (gather && (warp == 2 || warp == 3)) {
    // --------------- gather of this CTA's 128 routed A rows ---------------
    constexpr int kLag = MOE_GATHER_LAG_PAIR;
    static_assert(kLag >= 0 && kLag < STAGES, "gather lag below the ring depth");
    const int gt = tid - 64;
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0, arrived = 0;
    bool ok = true;
    const char *xs = static_cast<const char *>(P.gather_src);
    const int64_t row_bytes = (int64_t)P.K * 2;
    // stage s is full on the even CTA's barrier
    auto arrive_full = [&](int s) {
      if (rank == 0) mbar_arrive(&full_bar[s]);
      else mbar_arrive_cluster(mapa_shared(smem_u32(&full_bar[s]), 0));
    };
    while (ok && sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      const bool routed = tl.g < P.n_routed;
      GatherRows gr;
      if (routed) gr.load(P, s_off[tl.g], s_rows[tl.g], tl.m * PM + (int)rank * BM, gt);
      else gr.clear();
      for (int kb = kb0; kb < kb1; ++kb) {
        // lane 0 waits for the stage to be free, the warp follows it
        int okw = 1;
        if (lane == 0) okw = mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, s_limit) ? 1 : 0;
        __syncwarp();
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        if (routed) gr.issue(smem_u32(smem + (size_t)stage * stage_bytes), gt, kb, xs, row_bytes);
        cp_async_commit();
        ++issued;
        if (issued - arrived > kLag) {
          cp_async_wait<kLag>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) arrive_full((int)(arrived % STAGES));   // one arrival per warp
          ++arrived;
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    for (; arrived < issued; ++arrived)
      if (lane == 0) arrive_full((int)(arrived % STAGES));
  } else if (warp >= 4) {
    // -------------------------------- epilogue --------------------------------
    const int ew = warp - 4;
    const int r_cta = ew * 32 + lane;                 // row within this CTA's half
    uint8_t *stg = smem + (size_t)STAGES * stage_bytes + (size_t)ew * kStageBytesPerWarp;
    const uint32_t acce_even0 = mapa_shared(smem_u32(&acce_bar[0]), 0);
    const uint32_t acce_even1 = mapa_shared(smem_u32(&acce_bar[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    while (sc.next(tile, kb0, kb1, part)) {
      const Tile tl = decode_tile(P.reverse ? s_prefix[P.G] - 1 - tile : tile, s_prefix, P.G, P.nt);
      // (warp-uniform exits: the epilogue's TMEM loads and stores are warp-wide)
      if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[acc], acc_phase, &s_abort, P.err, s_limit))) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * kAccCols) + ((uint32_t)(ew * 32) << 16);
      const bool in_tail = sk && tile >= sc.dp_limit;
      if (P.kgroup) {
        // weight gradient tile: rows of group g's [M, N] output (split at split_m)
        const int row = tl.m * PM + (int)rank * BM + r_cta;
        const bool zero = s_rows[tl.g] == 0;
        float *dst = nullptr;
        if (row < P.M)
          dst = row < P.split_m
                    ? reinterpret_cast<float *>(P.out) + ((int64_t)tl.g * P.split_m + row) * P.N
                    : reinterpret_cast<float *>(P.out2) +
                          ((int64_t)tl.g * (P.M - P.split_m) + row - P.split_m) * P.N;
        // the warp's 32 rows by TMA stores when they lie in one output part
        const int row0w = tl.m * PM + (int)rank * BM + ew * 32;
        const CUtensorMap *om = nullptr;
        int64_t orow = 0;
        if (P.tma_store && row0w + 32 <= P.M) {
          if (row0w + 32 <= P.split_m) {
            om = &map_out;
            orow = (int64_t)tl.g * P.split_m + row0w;
          } else if (row0w >= P.split_m) {
            om = &map_out2;
            orow = (int64_t)tl.g * (P.M - P.split_m) + row0w - P.split_m;
          }
        }
        epilogue_wgrad(P, taddr, zero, dst, tl.n * P.bnh, stg, lane, om, orow);
      } else if (in_tail && kb0 > 0) {
        sk_write(P, 2 * pair + (int)rank, r_cta, taddr);        // a later piece of the tile
      } else {
        const bool routed = tl.g < P.n_routed;
        const int r_in = (int)rank * BM + r_cta;
        const bool valid = tl.m * PM + r_in < s_rows[tl.g];
        const int64_t out_row = (routed ? (int64_t)s_off[tl.g]
                                        : P.out_static_base + (int64_t)(tl.g - P.n_routed) * P.rows_static) +
                                (int64_t)tl.m * PM + r_in;
        const int col0 = tl.n * P.bnh;
        const int dest = (EPI == kEpiScaleAdd && valid) ? add_dest(P, routed, out_row, tl.m * PM + r_in) : -1;
        if (in_tail && kb1 < KB) {                              // finalizer of a split tile
          const Fixup F{P.sk_part, &sc, pair + 1, sc.contributors_end(tile), 2, (int)rank, r_cta};
          if (!__all_sync(0xffffffffu, sk_wait(P, F, &s_abort, s_limit))) break;
          epilogue_tile<EPI>(P, taddr, valid, routed, out_row, col0, stg, lane, 0, &F, dest, &map_out);
          sk_done(P, F);
        } else {
          epilogue_tile<EPI>(P, taddr, valid, routed, out_row, col0, stg, lane, 0, nullptr, dest, &map_out);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? acce_even0 : acce_even1);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (P.tma_store && lane == 0) bulk_wait_all();     // this warp's TMA stores written
  }

  tc_fence_before();
  cluster_sync_all();              // neither CTA leaves while the pair may still touch it
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}

// ------------------ the kernel, token-N version (CTA pairs) ------------------
// The forward expert GEMMs (kEpiRelu, kEpiSwiglu, kEpiScale, kEpiScaleAdd)
// with the operands' roles swapped: the weights are the MMA's M side (256
// rows a pair tile, 128 a CTA) and a group's token rows its N side, in tiles
// of at most 256 rows cut to multiples of 32.  A group of n rows runs
// ceil(n / 256) token tiles of nearly equal width, so a tile computes at most
// 31 padding rows: an expert of 277 rows costs 288 rows of MMA work instead
// of 384 on 128-row tiles or 512 on 256-row tiles.  The accumulator holds one
// weight row (output column) per TMEM lane and one token per column; the
// epilogue transposes it through shared memory into whole output rows.
//   A (weights): ReLU and the down-projection take 128 consecutive rows of W
//     per CTA; SwiGLU takes 64 rows of W1 (gate) and the same 64 rows of W3
//     (up), so a CTA's accumulator holds both halves of its 64 outputs.
//   B (tokens): the tile's N rows, N / 2 per CTA, in one TMA load: a tensor
//     map per box height (16, 32, ..., 128 rows), so a k-block costs one
//     copy of the weights (two for SwiGLU) and one of the tokens.  (Each TMA
//     instruction has a fixed cost: with 16-row boxes the tensor pipe sat
//     idle 64% of the time on the DeepSeek-V2 shape, with one box 42%.)
// Tiles run group by group, weight tile outer and token tile inner, so the
// pairs working at once share a weight tile in L2; they are dealt
// round-robin (no stream-K tail).
constexpr int kTnTokBox = 16;            // token box heights are multiples of this
// stages of two k-blocks (one 3-D copy each) for large token-N GEMMs;
// token-N epilogue: whole 32-column x NT-token pieces of the output leave
// through TMA stores from the staging buffer (a tile's ragged last tokens
// by plain stores); 0: plain stores throughout
#ifndef MOE_TN_TMA_STORE
#define MOE_TN_TMA_STORE 1
#endif
// the same for the single-CTA and CTA-pair kernels' bf16 forward outputs
#ifndef MOE_PAIR_TMA_STORE
#define MOE_PAIR_TMA_STORE 1
#endif
// MOE_TN_BK2=0 at build time: six stages of one k-block
#ifndef MOE_TN_BK2
#define MOE_TN_BK2 1
#endif
constexpr int kTnBoxes = 8;              // one tensor map per height 16, 32, ..., 128
constexpr int kTnMaxN = 256;             // token rows per tile (the MMA's N)
constexpr int kTnGran = 32;              // tile widths are multiples of this
constexpr int kTnStgBytes = 2304;        // per epilogue warp: 33 rows of 64 bytes (+ pad)
constexpr int kTnXchBytes = 16384;       // SwiGLU: 2 warp pairs x 2 buffers x 4 KB

struct TnTile {
  int g, wt, n0, n, valid;               // group, weight tile, first token, MMA N, rows stored
};

// The token-N kernel's tensor maps: token rows of the routed segments (x_perm
// or h) and of the static groups (x or h), one map per box height
// 16 (i + 1) rows, 3-D (one copy brings the stage's BKS k-blocks); the
// weights: 3-D boxes of 128 rows, or (SwiGLU) 2-D boxes of 64 rows of W1 and
// of W3, which must interleave k-block by k-block.
struct TnMaps {
  CUtensorMap tok[kTnBoxes];
  CUtensorMap tok_static[kTnBoxes];
  CUtensorMap w, w3;
  CUtensorMap out;            // output rows, boxes of 32 columns x NT tokens (tma_store)
};

// tiles per group: weight tiles x token tiles of at most maxn rows
__device__ __forceinline__ int tn_token_tiles(int rows, int maxn) { return (rows + maxn - 1) / maxn; }

__device__ __forceinline__ TnTile tn_decode(int tile, const int *prefix, const int *rows, int G,
                                            int maxn) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {                      // largest g with prefix[g] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  TnTile t;
  t.g = lo;
  const int r = rows[lo];
  const int nn = tn_token_tiles(r, maxn);
  const int width = ((r + nn - 1) / nn + kTnGran - 1) / kTnGran * kTnGran;
  const int local = tile - prefix[lo];
  t.wt = local / nn;
  t.n0 = (local - t.wt * nn) * width;
  t.valid = min(width, r - t.n0);
  t.n = (t.valid + kTnGran - 1) / kTnGran * kTnGran;        // the last tile may be narrower
  return t;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// NT tokens x this warp's 32 output columns (lane l: column col_base + l;
// vals[i]: token tok0 + i of the tile) into the output rows, as 16-byte
// pieces of whole 64-byte row segments.  Adjacent lanes first trade halves
// (even lanes keep columns l, l+1 of the first NT/2 tokens, odd lanes
// columns l-1, l of the others) and write packed bf16 pairs into a staging
// area of one 64-byte row per token (the second half of the tokens one row
// further on, so that the two halves fall on different banks); then every
// lane reads back 16-byte pieces and stores them.  Tokens at or past
// `valid` and columns past the output width are not written.  kEpiScaleAdd
// adds the piece into the token's row of y (routed: add_rows[out row];
// static group: its token index) with bf16 vector reductions instead.
template <int NT, int EPI>
__device__ __forceinline__ void store_tn(const Params &P, const float (&vals)[NT], int64_t row0,
                                         int tok0, int valid, bool routed, int64_t static_tok0,
                                         int col_base, uint8_t *stg, int lane,
                                         const CUtensorMap *omap, int &spar) {
  __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(P.out);
  const int64_t ld = P.N;
  const bool odd = (lane & 1) != 0;
  // a whole box of NT tokens x 32 columns: packed into the staging buffer as
  // NT rows of 64 bytes and stored by one TMA store (two buffers in turn
  // when they fit, so the next chunk need not wait for this store)
  constexpr int kBoxBytes = NT * 64;
  constexpr int kBufs = 2 * kBoxBytes <= kTnStgBytes ? 2 : 1;
  if (EPI != kEpiScaleAdd && MOE_TN_TMA_STORE && P.tma_store && tok0 + NT <= valid &&
      col_base + 32 <= P.N) {
    uint8_t *buf = stg + (kBufs == 2 ? spar * kBoxBytes : 0);
    if (lane == 0) {                                  // the store that read this buffer last is done reading
      if (kBufs == 2) bulk_wait_read<1>();
      else bulk_wait_read<0>();
    }
    __syncwarp();
    uint32_t *sw = reinterpret_cast<uint32_t *>(buf);
#pragma unroll
    for (int i = 0; i < NT / 2; ++i) {
      const float send = odd ? vals[i] : vals[NT / 2 + i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      const uint32_t w = odd ? pack_bf16x2(recv, vals[NT / 2 + i]) : pack_bf16x2(vals[i], recv);
      sw[(odd ? NT / 2 + i : i) * 16 + (lane >> 1)] = w;
    }
    fence_proxy_async_smem();                         // the tensor store reads through the async proxy
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(omap, buf, col_base, (int)(row0 + tok0));
      bulk_commit();
    }
    spar ^= kBufs - 1;
    return;
  }
  if (MOE_TN_TMA_STORE && P.tma_store) {              // the staging buffer is read no more
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }
  uint32_t *sw = reinterpret_cast<uint32_t *>(stg);
#pragma unroll
  for (int i = 0; i < NT / 2; ++i) {
    const float send = odd ? vals[i] : vals[NT / 2 + i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const uint32_t w = odd ? pack_bf16x2(recv, vals[NT / 2 + i]) : pack_bf16x2(vals[i], recv);
    const int srow = odd ? NT / 2 + i + 1 : i;
    sw[srow * 16 + (lane >> 1)] = w;
  }
  __syncwarp();
#pragma unroll
  for (int it = 0; it < NT / 8; ++it) {
    const int n = it * 8 + (lane >> 2), p = lane & 3;
    const int srow = n + (n >= NT / 2 ? 1 : 0);
    const uint4 w = *reinterpret_cast<const uint4 *>(stg + srow * 64 + p * 16);
    const int tok = tok0 + n;
    const int col = col_base + p * 8;
    if (tok < valid && col < P.N) {
      if constexpr (EPI == kEpiScaleAdd) {
        const int64_t dest = routed ? (int64_t)P.add_rows[row0 + tok] : static_tok0 + tok;
        if (dest >= 0 && dest < P.src_rows) red_add_bf16x8(out + dest * ld + col, w);
        else raise_error(P.err, kErrBadIndex);
      } else {
        *reinterpret_cast<uint4 *>(out + (row0 + tok) * ld + col) = w;
      }
    }
  }
  __syncwarp();
}

// Epilogue of one token-N tile, this warp's 32 TMEM lanes (weight rows) x
// the tile's tokens, 32 tokens (TMEM columns) at a time.  SwiGLU: warps
// ew and ew + 2 hold the gate and up rows of the same 32 outputs; they trade
// half of each 32-token chunk through `xch` (two buffers, so one barrier of
// the two warps per chunk suffices) and each stores 16 tokens of h.
template <int EPI>
__device__ __forceinline__ void epilogue_tn(const Params &P, uint32_t taddr, const TnTile &tl,
                                            bool routed, int64_t row0, int64_t static_tok0,
                                            int col_base, uint8_t *stg, float *xch, int ew, int lane,
                                            int &xpar, const CUtensorMap *omap, int &spar) {
  for (int c = 0; c < tl.n / 32; ++c) {
    if (32 * c >= tl.valid) break;                            // the same for the whole tile
    float v[32];
    acc_cols(taddr, 32 * c, nullptr, v);
    if constexpr (EPI == kEpiSwiglu) {
      const int pr = ew & 1;                                  // warps pr (gate) and pr + 2 (up)
      const bool gate_warp = ew < 2;
      float *xg = xch + (size_t)(pr * 2 + xpar) * 1024;       // gate values of tokens 16..31
      float *xu = xg + 512;                                   // up values of tokens 0..15
      if (gate_warp) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xg[i * 32 + lane] = v[16 + i];
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xu[i * 32 + lane] = v[i];
      }
      named_bar_sync(1 + pr, 64);
      float h[16];
      if (gate_warp) {
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = silu_f(v[i]) * xu[i * 32 + lane];
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float g = xg[i * 32 + lane];
          h[i] = silu_f(g) * v[16 + i];
        }
      }
      xpar ^= 1;
      store_tn<16, EPI>(P, h, row0, 32 * c + (gate_warp ? 0 : 16), tl.valid, routed, static_tok0,
                        col_base, stg, lane, omap, spar);
    } else {
      if constexpr (EPI == kEpiRelu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], 0.0f);
      } else {
        // gated rows: the gate of token 32c + i (routed groups; static: 1)
        float gm = 1.0f;
        if (routed && 32 * c + lane < tl.valid) gm = P.row_gate[row0 + 32 * c + lane];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= __shfl_sync(0xffffffffu, gm, i);
      }
      store_tn<32, EPI>(P, v, row0, 32 * c, tl.valid, routed, static_tok0, col_base, stg, lane,
                        omap, spar);
    }
  }
}

template <int EPI, int BKS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_tn_kernel(const __grid_constant__ TnMaps M, const Params P) {
  constexpr bool kSwiglu = EPI == kEpiSwiglu;
  constexpr int kMaxN = kTnMaxN;                                // token rows per tile
  constexpr int STAGES = BKS == 2 ? kPairStages2 : kPairStages;
  constexpr uint32_t kWBytes = BM * BK * 2;                     // weights: 16 KB a k-block and CTA
  constexpr uint32_t kTokBytes = (kMaxN / 2) * BK * 2;          // token rows: up to 16 KB
  constexpr uint32_t stage_bytes = BKS * (kWBytes + kTokBytes);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int s_prefix[kMaxGroups + 1];
  __shared__ int s_off[kMaxGroups];
  __shared__ int s_rows[kMaxGroups];
  __shared__ __align__(8) uint64_t full_bar[kPairStages];
  __shared__ __align__(8) uint64_t empty_bar[kPairStages];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ uint64_t s_limit_sh;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (tid == 32) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full_bar[st], 1);                     // the even CTA's expect_tx arrival
      mbar_init(&empty_bar[st], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf_bar[a], 1);
      mbar_init(&acce_bar[a], 2 * 4 * 32);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  if (tid == 0) {
    tma_prefetch_map(&M.w);
    if (kSwiglu) tma_prefetch_map(&M.w3);
  }
  pdl_wait();              // what earlier kernels wrote is visible from here on
  pdl_trigger();
  if (tid == 0) s_limit_sh = wait_limit_ns(P.err);
  if (warp == 0) {
    // group table: rows of each group and the tile prefix (weight tiles x token tiles)
    int carry = 0;
    for (int base = 0; base < P.G; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < P.G) {
        int off = 0, rows = 0;
        if (g < P.n_routed) {
          off = P.offsets[g];
          rows = P.offsets[g + 1] - off;
          if (rows < 0 || off < 0 || (int64_t)off + rows > P.seg_rows) {
            raise_error(P.err, kErrBadIndex);
            rows = 0;
            off = 0;
          }
        } else {
          rows = (int)P.rows_static;
        }
        s_off[g] = off;
        s_rows[g] = rows;
        tiles = tn_token_tiles(rows, kMaxN) * P.nt;
      }
      int x = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (g < P.G) s_prefix[g] = carry + x - tiles;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_prefix[P.G] = carry;
  }
  tc_fence_before();
  cluster_sync_all();              // barriers of both CTAs initialised before any remote use
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const uint64_t s_limit = s_limit_sh;
  const int KB = P.K / (BK * BKS);                     // stages of K per tile
  const int total = s_prefix[P.G];

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += npairs) {
      const TnTile tl = tn_decode(tile, s_prefix, s_rows, P.G, kMaxN);
      const bool routed = tl.g < P.n_routed;
      const int half = tl.n / 2;                       // this CTA's token rows: one box
      const CUtensorMap *mt = routed ? &M.tok[half / kTnTokBox - 1] : &M.tok_static[half / kTnTokBox - 1];
      const int tok_row =
          (int)((routed ? (int64_t)s_off[tl.g]
                        : P.a_static_base + (int64_t)(tl.g - P.n_routed) * P.a_static_stride) +
                tl.n0 + (int64_t)rank * half);
      const int w_row = kSwiglu ? tl.g * P.N + tl.wt * 128 + (int)rank * 64
                                : tl.g * P.N + tl.wt * 256 + (int)rank * 128;
      const uint32_t tx = 2u * BKS * (kWBytes + (uint32_t)half * BK * 2);
      const int kz = 0;                                // 3-D maps: k-block coordinate below
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
        uint8_t *sa = smem + (size_t)stage * stage_bytes;
        uint8_t *sb = sa + BKS * kWBytes;
        const uint32_t fb = smem_u32(&full_bar[stage]) & 0xFEFFFFFFu;   // the even CTA's barrier
        if (rank == 0) {
          mbar_expect_tx(&full_bar[stage], tx);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        (void)kz;
        if (kSwiglu) {
#pragma unroll
          for (int q = 0; q < BKS; ++q) {
            const int kx = (kb * BKS + q) * BK;
            tma_load_2d_pair(sa + q * kWBytes, &M.w, fb, kx, w_row);
            tma_load_2d_pair(sa + q * kWBytes + kWBytes / 2, &M.w3, fb, kx, w_row);
          }
        } else {
          tma_load_3d_pair(sa, &M.w, fb, 0, w_row, kb * BKS);            // BKS tiles of 16 KB
        }
        tma_load_3d_pair(sb, mt, fb, 0, tok_row, kb * BKS);               // BKS tiles of half rows
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && rank == 0) {
      for (int st = 0; st < STAGES; ++st)
        if (armed & (1u << st)) mbar_wait_drain(&full_bar[st], (armed_parity >> st) & 1u);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------ MMA issuer (even CTA only) ------------------------
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += npairs) {
      const TnTile tl = tn_decode(tile, s_prefix, s_rows, P.G, kMaxN);
      const uint32_t idesc = idesc_bf16(2 * BM, tl.n);
      if (!mbar_wait(&acce_bar[acc], acc_phase ^ 1u, &s_abort, P.err, s_limit)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait<true>(&full_bar[stage], phase, &s_abort, P.err, s_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + (size_t)stage * stage_bytes);
        const uint32_t b_addr = a_addr + BKS * kWBytes;
        const uint32_t b_chunk = (uint32_t)(tl.n / 2) * BK * 2;   // token tiles lie back to back
#pragma unroll
        for (int q = 0; q < BKS; ++q) {
#pragma unroll
          for (int k = 0; k < BK / kUmmaK; ++k)
            umma_bf16_pair(d_tmem, sw128_desc(a_addr + q * kWBytes + k * kUmmaK * 2),
                           sw128_desc(b_addr + q * b_chunk + k * kUmmaK * 2), idesc,
                           (kb > 0 || q > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit_pair_both(&empty_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit_pair_both(&accf_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    umma_commit_pair_local(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  } else if (warp >= 4) {
    // -------------------------------- epilogue --------------------------------
    const int ew = warp - 4;                           // TMEM lanes 32 ew .. 32 ew + 31
    uint8_t *stg = smem + (size_t)STAGES * stage_bytes + (size_t)ew * kTnStgBytes;
    float *xch = reinterpret_cast<float *>(smem + (size_t)STAGES * stage_bytes + 4 * kTnStgBytes);
    const uint32_t acce_even0 = mapa_shared(smem_u32(&acce_bar[0]), 0);
    const uint32_t acce_even1 = mapa_shared(smem_u32(&acce_bar[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    int xpar = 0, spar = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const TnTile tl = tn_decode(tile, s_prefix, s_rows, P.G, kMaxN);
      // (warp-uniform exits: the epilogue's TMEM loads and stores are warp-wide)
      if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[acc], acc_phase, &s_abort, P.err, s_limit))) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * kAccCols) + ((uint32_t)(ew * 32) << 16);
      const bool routed = tl.g < P.n_routed;
      const int64_t row0 = (routed ? (int64_t)s_off[tl.g]
                                   : P.out_static_base + (int64_t)(tl.g - P.n_routed) * P.rows_static) +
                           tl.n0;
      const int col_base = kSwiglu ? tl.wt * 128 + (int)rank * 64 + 32 * (ew & 1)
                                   : tl.wt * 256 + (int)rank * 128 + 32 * ew;
      epilogue_tn<EPI>(P, taddr, tl, routed, row0, (int64_t)tl.n0, col_base, stg, xch, ew, lane, xpar,
                       &M.out, spar);
      tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? acce_even0 : acce_even1);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();                 // this warp's TMA stores written before the CTA ends
  }

  tc_fence_before();
  cluster_sync_all();              // neither CTA leaves while the pair may still touch it
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}

}  // namespace

// ------------------------------- host helpers --------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous), box [box_outer, 64].
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (outer == 0) outer = 1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view {64 columns, rows, K / 64 k-blocks} of a bf16 matrix [rows][K]
// (strides: K * 2 bytes between rows, 128 bytes between k-blocks), box
// {64, box_rows, chunks}: one copy brings `chunks` consecutive k-blocks of
// box_rows rows, landing as `chunks` [box_rows][64] tiles one after another,
// each 128-byte swizzled like a 2-D box.
bool make_map3(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint32_t box_rows,
               uint32_t chunks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (rows == 0) rows = 1;
  cuuint64_t dims[3] = {(cuuint64_t)BK, rows, K / BK};
  cuuint64_t strides[2] = {K * 2, (cuuint64_t)BK * 2};
  cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [outer][inner] (inner contiguous) in boxes of box_outer
// rows x box_inner columns, no swizzle: the token-N epilogue's TMA stores
// (rows of box_inner * 2 bytes in shared memory).
bool make_map_box(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor [outer][inner] (inner contiguous) in boxes of 32 rows x
// 32 columns (128 bytes), 128-byte swizzled: the weight-gradient epilogue's
// TMA stores from its swizzled staging.
bool make_map_f32(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || outer == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

namespace {

template <int EPI>
cudaError_t launch_epi(const Params &P, const CUtensorMap &ma,
                       const CUtensorMap &mas, const CUtensorMap &mb, const CUtensorMap &mb3,
                       const CUtensorMap &mo, int grid, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<EPI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(grouped_gemm_kernel<EPI>, grid, kThreads, smem, s, ma, mas, mb, mb3, mo, P);
}

// CTA-pair launch: as many 2-CTA clusters as fit at once (one CTA per SM),
// fewer when there are fewer tiles.
template <int EPI, int BKS>
cudaError_t launch_pair(const Params &P, const CUtensorMap &ma, const CUtensorMap &mas,
                        const CUtensorMap &mb, const CUtensorMap &mb3, const CUtensorMap &mo,
                        const CUtensorMap &mo2, int64_t max_tiles, size_t smem, cudaStream_t s) {
  auto kern = grouped_gemm_pair_kernel<EPI, BKS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  static int max_clusters[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int dev = 0;
  cudaGetDevice(&dev);
  int &mc = max_clusters[dev & 7];
  if (mc == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = device_sms() / 2;
    }
    mc = n;
  }
  const int64_t want = P.sk_part ? mc : std::min<int64_t>(mc, max_tiles);
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(want, kSkSlots / 2));
  return launch_kernel(kern, 2 * pairs, kThreads, smem, s, ma, mas, mb, mb3, mo, mo2, P);
}

// Token-N launch: as many 2-CTA clusters as fit at once, fewer when there are
// fewer tiles.
template <int EPI, int BKS>
cudaError_t launch_tn(const Params &P, const TnMaps &maps, int64_t max_tiles, size_t smem,
                      cudaStream_t s) {
  auto kern = grouped_gemm_tn_kernel<EPI, BKS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  static int max_clusters[8][4] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int &mc = max_clusters[dev & 7][(EPI == kEpiSwiglu ? 2 : 0) + (BKS - 1)];
  if (mc == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = device_sms() / 2;
    }
    mc = n;
  }
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(mc, max_tiles));
  return launch_kernel(kern, 2 * pairs, kThreads, smem, s, maps, P);
}

}  // namespace

cudaError_t launch_grouped_gemm(const GroupedGemm &g, cudaStream_t s) {
  Params P{};
  P.epi = g.epi;
  P.K = g.K;
  P.N = g.N;
  if (swiglu_b(g.epi)) {
    P.bn = 256;
    P.bnh = 128;
  } else if (g.epi == kEpiStoreF32) {
    P.bn = std::min(256, std::max(32, (g.N + 31) / 32 * 32));
    P.bnh = P.bn;
  } else {
    P.bn = 256;
    P.bnh = 256;
  }
  P.nt = (g.N + P.bnh - 1) / P.bnh;
  P.n_routed = g.n_routed;
  P.n_static = g.n_static;
  P.G = g.n_routed + g.n_static;
  P.rows_static = g.rows_static;
  P.a_static_base = g.a_static_base;
  P.a_static_stride = g.a_static_stride;
  P.out_static_base = g.out_static_base;
  P.a_rows = g.a_rows;
  P.seg_rows = g.gather_rows ? g.max_routed_rows : g.a_rows;
  P.offsets = g.offsets;
  P.out = g.out;
  P.row_gate = g.row_gate;
  P.bias = g.bias;
  P.ksplit = std::max(1, g.ksplit);
  P.split_stride = g.split_stride;
  P.b_mn = g.b_mn;
  P.b_kb_split = g.b_mn ? (g.b_kb_split > 0 ? g.b_kb_split : g.K / BK) : 0;
  P.b_krows = g.b_krows;
  P.kgroup = g.kgroup;
  P.M = g.M;
  P.kseg = g.kseg;
  P.split_m = g.out2 ? g.split_m : g.M;
  P.out2 = g.out2;
  P.aux = g.aux;
  P.aux_ld = g.aux_ld;
  P.dg_part = g.dg_part;
  P.dg_nt = g.dg_nt;
  P.aux2 = g.aux2;
  P.aux2_ld = g.aux2_ld;
  P.add_rows = g.add_rows;
  // stream-K tail for the expert GEMMs (not with the router's K split or K groups)
  const bool sk = MOE_STREAM_K && P.ksplit == 1 && !g.kgroup && g.n_routed > 0 && g.sk_part &&
                  g.sk_flags;
  P.sk_part = sk ? g.sk_part : nullptr;
  P.sk_flags = sk ? g.sk_flags : nullptr;
  P.reverse = g.reverse;
  P.gather_rows = g.gather_rows;
  P.gather_src = g.gather_src;
  P.src_rows = g.src_rows;
  if (g.gather_rows && (!g.gather_src || g.epi == kEpiStoreF32 || g.n_routed == 0 || g.kgroup))
    return cudaErrorInvalidValue;
  P.err = g.err;
  if (P.G <= 0 || P.G > kMaxGroups || P.bn > 256 || g.K % BK != 0) return cudaErrorInvalidValue;
  if (g.ksplit > 1 && (g.epi != kEpiStoreF32 || g.n_routed != 0)) return cudaErrorInvalidValue;
  if ((g.epi == kEpiDActRelu || g.epi == kEpiDActSwiglu) && (!g.aux || !g.row_gate))
    return cudaErrorInvalidValue;
  if (g.dg_part && (g.dg_nt != P.nt || (g.epi != kEpiDActRelu && g.epi != kEpiDActSwiglu) ||
                    (g.epi == kEpiDActSwiglu && !g.aux2)))
    return cudaErrorInvalidValue;
  // the folded combine: gates, the row -> token map, its range
  if (g.epi == kEpiScaleAdd && (!g.row_gate || !g.add_rows || g.src_rows <= 0 || g.N % 64 != 0))
    return cudaErrorInvalidValue;
  if (g.b_mn && (swiglu_b(g.epi) || g.kgroup || g.b_krows <= 0 || P.bn != 256))
    return cudaErrorInvalidValue;
  if (g.kgroup && (g.epi != kEpiStoreF32 || g.n_routed != 0 || !g.kseg || g.M <= 0 ||
                   (g.out2 && (g.split_m <= 0 || g.split_m >= g.M))))
    return cudaErrorInvalidValue;

  // token-N tiles (weights on the MMA's M side) for the forward expert GEMMs
  // of short groups
  const bool tn_epi = g.epi == kEpiRelu || g.epi == kEpiSwiglu || g.epi == kEpiScale ||
                      g.epi == kEpiScaleAdd;
  if (tn_epi && !g.kgroup && g.n_routed > 0 && !g.gather_rows && !g.b_mn && g.ksplit <= 1 &&
      g.max_routed_rows / g.n_routed < MOE_TN_MAX_ROWS) {
    const bool swiglu = g.epi == kEpiSwiglu;
    const int maxn = kTnMaxN;
    Params Q = P;
    Q.nt = swiglu ? (g.N + 127) / 128 : (g.N + 255) / 256;     // weight tiles per group
    Q.sk_part = nullptr;
    Q.sk_flags = nullptr;
    const double macs_tn = (double)(g.max_routed_rows + (int64_t)g.n_static * g.rows_static) * g.N *
                           g.K * (swiglu ? 2 : 1);
    const bool bk2_tn = MOE_TN_BK2 && g.K % (2 * BK) == 0 && macs_tn >= 2e11;
    const uint32_t chunks = bk2_tn ? 2u : 1u;
    TnMaps maps;
    for (int i = 0; i < kTnBoxes; ++i) {
      const uint32_t h = (uint32_t)(kTnTokBox * (i + 1));
      if (!make_map3(&maps.tok[i], g.a, (uint64_t)g.K, (uint64_t)g.a_rows, h, chunks))
        return cudaErrorInvalidValue;
      if (!make_map3(&maps.tok_static[i], g.a_static ? g.a_static : g.a, (uint64_t)g.K,
                     (uint64_t)(g.a_static ? g.a_static_rows : g.a_rows), h, chunks))
        return cudaErrorInvalidValue;
    }
    if (swiglu) {
      if (!make_map(&maps.w, g.b, (uint64_t)g.K, (uint64_t)g.b_rows, 64)) return cudaErrorInvalidValue;
      if (!make_map(&maps.w3, g.b3, (uint64_t)g.K, (uint64_t)g.b_rows, 64)) return cudaErrorInvalidValue;
    } else {
      if (!make_map3(&maps.w, g.b, (uint64_t)g.K, (uint64_t)g.b_rows, 128, chunks))
        return cudaErrorInvalidValue;
      maps.w3 = maps.w;
    }
    // TMA stores of the outputs: boxes of 32 columns x 16 (SwiGLU) or 32 tokens
    Q.tma_store = 0;
    if (MOE_TN_TMA_STORE && g.epi != kEpiScaleAdd && g.out_rows > 0 && g.out_rows < ((int64_t)1 << 31) &&
        g.N % 32 == 0 &&
        make_map_box(&maps.out, g.out, (uint64_t)g.N, (uint64_t)g.out_rows, 32, swiglu ? 16u : 32u))
      Q.tma_store = 1;
    const int64_t tt_routed = (g.max_routed_rows + maxn - 1) / maxn + g.n_routed;
    const int64_t tt_static = (int64_t)g.n_static * ((g.rows_static + maxn - 1) / maxn);
    const int64_t max_tiles = (tt_routed + tt_static) * Q.nt;
    const bool bk2 = bk2_tn;
    const size_t stage = (size_t)(bk2 ? 2 : 1) * ((size_t)kABytes + (size_t)(maxn / 2) * BK * 2);
    const size_t nstages = bk2 ? (size_t)kPairStages2 : (size_t)kPairStages;
    const size_t tsmem = nstages * stage + 1024 + 4 * (size_t)kTnStgBytes +
                         (swiglu ? (size_t)kTnXchBytes : 0);
#define MOE_TN_CASE(E_)                                                                  \
  case E_:                                                                               \
    return bk2 ? launch_tn<E_, 2>(Q, maps, max_tiles, tsmem, s)                          \
               : launch_tn<E_, 1>(Q, maps, max_tiles, tsmem, s);
    switch (g.epi) {
      MOE_TN_CASE(kEpiRelu)
      MOE_TN_CASE(kEpiSwiglu)
      MOE_TN_CASE(kEpiScale)
      MOE_TN_CASE(kEpiScaleAdd)
      default: return cudaErrorInvalidValue;
    }
#undef MOE_TN_CASE
  }

  // CTA pairs for the expert GEMMs whose groups are long enough that 256-row
  // tiles waste little (average routed rows per expert >= MOE_PAIR_MIN_ROWS),
  // and for weight gradients of at least 256 rows
  const bool pair = P.bn == 256 &&
                    ((!g.kgroup && g.n_routed > 0 && g.max_routed_rows / g.n_routed >= MOE_PAIR_MIN_ROWS) ||
                     (g.kgroup && g.M >= 2 * BM && MOE_PAIR_WGRAD));
  CUtensorMap ma, mas, mb, mb3, mo;
  // bf16 forward outputs: whole 32-row x 64-column pieces by TMA stores
  // (boxes of the 128-byte-swizzled staging)
  P.tma_store = 0;
  if (MOE_PAIR_TMA_STORE && (g.epi == kEpiRelu || g.epi == kEpiSwiglu || g.epi == kEpiScale) &&
      !g.kgroup && g.out_rows > 0 && g.out_rows < ((int64_t)1 << 31) && g.N % 64 == 0 &&
      make_map(&mo, g.out, (uint64_t)g.N, (uint64_t)g.out_rows, 32))
    P.tma_store = 1;
  // weight gradients (fp32, K groups) on CTA pairs: whole 32-row x 32-column
  // pieces by TMA stores, one map per output part (rows below split_m, and
  // the rest); a warp's rows never straddle the two when split_m is a
  // multiple of 32
  CUtensorMap mo2;
  if (MOE_PAIR_TMA_STORE && g.kgroup && pair && g.epi == kEpiStoreF32 && g.N % 4 == 0 &&
      (!g.out2 || P.split_m % 32 == 0) &&
      make_map_f32(&mo, g.out, (uint64_t)g.N, (uint64_t)P.G * P.split_m) &&
      (!g.out2 || make_map_f32(&mo2, g.out2, (uint64_t)g.N, (uint64_t)P.G * (g.M - P.split_m))))
    P.tma_store = 1;
  if (!g.out2 || !P.tma_store) mo2 = mo;
  const uint32_t box_b = (swiglu_b(g.epi) || pair) ? 128u : (uint32_t)P.bn;
  // K groups: A is [M, K] and B [N, K] with all groups' K columns side by side
  const uint64_t a_outer = g.kgroup ? (uint64_t)g.M : (uint64_t)g.a_rows;
  const uint64_t b_outer = g.kgroup ? (uint64_t)g.N : (uint64_t)g.b_rows;
  if (!make_map(&ma, g.a, (uint64_t)g.K, a_outer, BM)) return cudaErrorInvalidValue;
  if (!P.tma_store) {                                        // (not read)
    mo = ma;
    mo2 = ma;
  }
  if (!make_map(&mas, g.a_static && !g.kgroup ? g.a_static : g.a, (uint64_t)g.K,
                (uint64_t)(g.a_static && !g.kgroup ? g.a_static_rows : a_outer), BM))
    return cudaErrorInvalidValue;
  if (g.b_mn) {
    // B stored [K][N]: rows of N values, boxes of 64 N x 64 K
    if (!make_map(&mb, g.b, (uint64_t)g.N, (uint64_t)g.b_rows, 64)) return cudaErrorInvalidValue;
    if (!make_map(&mb3, g.b3 ? g.b3 : g.b, (uint64_t)g.N, (uint64_t)g.b_rows, 64))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map(&mb, g.b, (uint64_t)g.K, b_outer, box_b)) return cudaErrorInvalidValue;
    if (!make_map(&mb3, g.b3 ? g.b3 : g.b, (uint64_t)g.K, b_outer, box_b))
      return cudaErrorInvalidValue;
  }

  // grid: one CTA per SM, fewer when there are fewer tiles
  const int64_t mt_routed = (g.max_routed_rows + BM - 1) / BM + g.n_routed;
  const int64_t mt_static = (int64_t)g.n_static * (((g.kgroup ? g.M : g.rows_static) + BM - 1) / BM);
  const int64_t max_tiles = (mt_routed + mt_static) * P.nt * P.ksplit;
  // (with stream-K, every SM: a short problem's k-blocks are spread over all)
  const int grid = std::min(kSkSlots, (int)std::max<int64_t>(1, std::min<int64_t>(
                                          device_sms(), sk ? device_sms() : max_tiles)));
  // at least 120 KB so that one CTA (and one 512-column TMEM allocation) fits per SM
  const size_t smem = std::max<size_t>((size_t)kStages * (kABytes + (size_t)P.bn * BK * 2) + 1024 +
                                           4 * kStageBytesPerWarp,
                                       (size_t)120 * 1024);

  if (pair) {
    const int64_t pt_routed = (g.max_routed_rows + 2 * BM - 1) / (2 * BM) + g.n_routed;
    const int64_t pt_static =
        (int64_t)g.n_static * (((g.kgroup ? g.M : g.rows_static) + 2 * BM - 1) / (2 * BM));
    const int64_t pair_tiles = (pt_routed + pt_static) * P.nt;
    // stages of two k-blocks where K allows (no gather, K-major B, no K
    // groups) and the GEMM is large: measured 10% faster expert GEMMs on the
    // Mixtral shape and 5% on DeepSeekMoE's, 1% slower on the GShard shape's
    // 3.4e10-MAC GEMMs
    const double macs = (double)(g.max_routed_rows + (int64_t)g.n_static * g.rows_static) * g.N *
                        g.K * (swiglu_b(g.epi) ? 2 : 1);
    const bool bk2 = MOE_PAIR_BK128 && !g.kgroup && !g.b_mn && !g.gather_rows &&
                     g.K % (2 * BK) == 0 && macs >= 2e11;
    const size_t psmem = (bk2 ? (size_t)kPairStages2 * 2 : (size_t)kPairStages) *
                             (kABytes + (size_t)(P.bn / 2) * BK * 2) +
                         1024 + 4 * kStageBytesPerWarp;
#define MOE_PAIR_CASE(E_)                                                            \
  case E_:                                                                           \
    return bk2 ? launch_pair<E_, 2>(P, ma, mas, mb, mb3, mo, mo2, pair_tiles, psmem, s)   \
               : launch_pair<E_, 1>(P, ma, mas, mb, mb3, mo, mo2, pair_tiles, psmem, s);
    switch (g.epi) {
      MOE_PAIR_CASE(kEpiStoreF32)
      MOE_PAIR_CASE(kEpiRelu)
      MOE_PAIR_CASE(kEpiSwiglu)
      MOE_PAIR_CASE(kEpiScale)
      MOE_PAIR_CASE(kEpiPreRelu)
      MOE_PAIR_CASE(kEpiPreSwiglu)
      MOE_PAIR_CASE(kEpiDActRelu)
      MOE_PAIR_CASE(kEpiDActSwiglu)
      MOE_PAIR_CASE(kEpiScaleAdd)
      default: return cudaErrorInvalidValue;
    }
#undef MOE_PAIR_CASE
  }
#define MOE_ONE_CASE(E_)                                                             \
  case E_:                                                                           \
    return launch_epi<E_>(P, ma, mas, mb, mb3, mo, grid, smem, s);
  switch (g.epi) {
    MOE_ONE_CASE(kEpiStoreF32)
    MOE_ONE_CASE(kEpiRelu)
    MOE_ONE_CASE(kEpiSwiglu)
    MOE_ONE_CASE(kEpiScale)
    MOE_ONE_CASE(kEpiPreRelu)
    MOE_ONE_CASE(kEpiPreSwiglu)
    MOE_ONE_CASE(kEpiDActRelu)
    MOE_ONE_CASE(kEpiDActSwiglu)
    MOE_ONE_CASE(kEpiScaleAdd)
    default: return cudaErrorInvalidValue;
  }
#undef MOE_ONE_CASE
}

}  // namespace moe
