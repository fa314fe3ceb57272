// Chunked-prefill attention over the NVFP4 paged cache on the Blackwell tensor
// cores (tcgen05, fp32 accumulators in tensor memory).
//
// ("FlashInfer backend adds end-to-end NVFP4 KV cache support",
// implementation breakdown items 2-3: the prefill path reads the NVFP4 pages
// plus their FP8 block scales and writes FP8 output dequantized back to the
// model dtype.) Each sequence with q_len > 1 query tokens: query row r sits at
// position L - q_len + r and attends causally to keys 0..L-q_len+r of its
// paged cache; o = softmax(sm_scale * q K^T) V with K = E2M1 * E4M3 * k_scale
// and V likewise with v_scale.
//
// A CTA owns M = 128 rows: 128/G query tokens x the G query heads of one kv
// head (GQA), so every key chunk is read and dequantized once for all of them.
// Keys advance in chunks of 64:
//   S  = Q K^T   tcgen05.mma kind::f16, A = Q (f16, in TMEM), B = K chunk
//                (f16, 128B-swizzled shared tile, K-major), D = S (fp32, TMEM)
//   P  = exp2(S * scale - m) in fp32, split into f16 hi + lo (~22 bits: f16
//        alone misses the 2e-3 bound on outlier-heavy rows), written back to
//        TMEM over S's columns: per 16 keys, 8 columns of hi then 8 of lo
//   O += P V     A = P hi, then P lo (TMEM), B = V chunk (the same swizzled
//                tile layout read MN-major), D = O (fp32, TMEM)
// S/P buffers in TMEM: four (two at head size 256, where O and Q take 384 of
// the 512 columns), so S of later chunks is computed while the softmax of
// chunk c runs.
// E2M1 * E4M3 has at most 6 significant bits in [2^-10, 2688], so K and V are
// exact in f16; k_scale is folded into the logit scale and v_scale into the
// output. Q is scaled per row by a power of two putting max |q| in
// [2^14, 2^15), where f16 keeps every bf16 bit. The running max moves only when
// a chunk's max exceeds it by more than 2^8 (then O is rescaled in TMEM).
//
// Warp roles (20 warps):
//   0-3   Q rows into TMEM; softmax of keys [0, 32) of each chunk and epilogue
//         of O columns [0, D/2) (thread i = row i = TMEM lane i)
//   4     TMEM allocation; one thread issues the PV MMAs
//   5-8   K: dequantization of a chunk's raw NVFP4 pages into an f16 tile slot
//   9-12  V: the same for V (one code copy with K)
//   13    one thread issues the S MMAs
//   14-15 one thread each issues the bulk copies of K (V) pages into a raw
//         stage ring
//   16-19 softmax of keys [32, 64) and epilogue of O columns [D/2, D)
// The hot loops are kept rolled where unrolling buys little: with every role
// resident at once, an unrolled kernel outgrows the instruction cache.
// Every mbarrier wait is bounded; a wait that gives up raises NVFP4_DEV_TIMEOUT
// and makes the whole block stop, wait for its copies and MMAs, free its TMEM
// and return.
#include <mutex>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"
#include "nvfp4kv_tc.cuh"

namespace nvfp4kv {

namespace {
constexpr int kRows = 128;   // M of every MMA: (query token, head) rows per CTA
constexpr int kMaxSBufs = 4;  // S/P buffers in TMEM (at most)
constexpr int kMaxSlots = 3;  // f16 K (and V) tile slots (at most)
constexpr int kMaxRawStages = 3;  // raw page stages per K and V (at most)
// block ids of a CTA's pages held in shared memory (longer ranges read them
// from the block table as they go)
constexpr int kMaxIds = 4096;
constexpr int kThreads = 20 * 32;
constexpr int kMmaWarp = 4;    // TMEM allocation, PV MMAs
constexpr int kSWarp = 13;     // S MMAs
constexpr int kCopyWarp0 = 14; // K page copies (warp 15: V)
constexpr int kSoftmax1Warp0 = 16;  // second softmax group (warps 16-19)
constexpr int kKGroup0 = 5 * 32;  // first thread of the K warps
constexpr int kVGroup0 = 9 * 32;  // first thread of the V warps
constexpr uint32_t kBarSoftmax = 3, kBarCopy = 4;  // named barriers (256, 64 threads)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;
constexpr int kMaxPolls = 1 << 22;
#ifndef PREFILL_SUSPEND_NS
#define PREFILL_SUSPEND_NS 1000
#endif
#ifndef KV_WAIT
#define KV_WAIT kWaitSleep
#endif
#ifndef MMA_WAIT
#define MMA_WAIT kWaitSpin
#endif
#ifndef SM_WAIT
#define SM_WAIT kWaitSpin
#endif
// a CTA keeps the SM to itself (its TMEM allocation is the whole SM's)
constexpr size_t kMinSmem = 120 * 1024;

// Barrier slots.
enum : int {
  kBarKraw = 0,                   // [3] K raw stage filled (expect_tx)
  kBarVraw = kMaxRawStages,       // [3] V raw stage filled
  kBarKFull = 2 * kMaxRawStages,     // [3] K tile dequantized (128 arrivals)
  kBarVFull = kBarKFull + kMaxSlots, // [3] V tile dequantized (128 arrivals)
  kBarKEmpty = kBarVFull + kMaxSlots,  // [3] S MMAs that read the K tile done (commit)
  kBarVEmpty = kBarKEmpty + kMaxSlots, // [3] PV MMAs that read the V tile done (commit)
  kBarSFull = kBarVEmpty + kMaxSlots,  // [4] S chunk in TMEM (commit)
  kBarPFull = kBarSFull + kMaxSBufs, // [4][2] P of 16-key group g of both halves in TMEM (256 arrivals)
  kBarPFree = kBarPFull + 2 * kMaxSBufs, // [4] PV MMAs that read a P buffer done (commit)
  kBarQReady = kBarPFree + kMaxSBufs,  // Q rows in TMEM (128 arrivals)
  kBarRawEmpty = kBarQReady + 1,  // [2][3] K, V raw stage read by every dequant thread (128 arrivals)
  kBarSRead = kBarRawEmpty + 2 * kMaxRawStages,  // [4] S chunk read by both softmax groups (256 arrivals)
  kBarFin = kBarSRead + kMaxSBufs,  // every MMA issued done (2 commits)
  kNumBarriers = kBarFin + 1
};

template <int D, int BS, int FMT, bool QF>
struct PrefillShape {
  // keys per chunk: N of S = Q K^T and the K-extent of O += P V. S/P buffers
  // in TMEM: four, or two at head size 256 (where O and Q take 384 of the 512
  // columns); f16 K and V tile slots: three, or two at head size 256 (shared
  // memory).
  static_assert(!QF || (D == 256 && FMT == 0),
                "NVFP4 queries: head size 256 over the NVFP4 cache");
  static constexpr int kChunk = 64;
  // (QF: Q leaves TMEM for shared memory, making room for a third buffer)
  static constexpr int kSBufs = QF ? 3 : (D == 256 ? 2 : 4);
  // (QF: the K slots hold packed codes, 10 KB each, leaving room for three)
  static constexpr int kSlots = (D == 256 && !QF) ? 2 : 3;
  // raw page stages per K and V: three, or two for FP8 rows at head size 256
  static constexpr int kRawStages = (FMT && D == 256) ? 2 : 3;
  static constexpr int F = FMT ? D : D / 2 + D / 16;  // row bytes: NVFP4, or FP8 (FMT = 1)
  static constexpr int PAGE = BS * F;          // bytes of one (block, K|V, head) page
  static constexpr int PPC = kChunk >= BS ? kChunk / BS : 1;  // pages per chunk
  static constexpr int RAW = kChunk * F;       // cache bytes of a chunk (K or V)
  static constexpr int TILE = kChunk * D * 2;  // f16 tile of a chunk
  // QF: a K slot holds the chunk's E2M1 codes (K-major, 128B swizzle, one
  // 128-byte row per key) and one 512-byte scale tile per K step of 64
  static constexpr int KSTEPS = D / 64;
  static constexpr int KCODES = kChunk * D / 2;
  static constexpr int KTILE = QF ? KCODES + KSTEPS * 512 : TILE;
  // QF: the Q tile, codes (128 rows x 128 bytes, swizzled as K) then its scale tiles
  static constexpr int QCODES = kRows * D / 2;
  static constexpr int QTILE = QF ? QCODES + KSTEPS * 512 : 0;
  // TMEM columns: O [0, D), S/P buffers [D, D + kSBufs chunk), then Q (D/2, f16)
  // or, QF, the scale factors: Q's (4 columns per K step), then each K slot's
  static constexpr uint32_t kColO = 0, kColS = D, kColQ = D + kSBufs * kChunk;
  static constexpr uint32_t kColSFA = kColQ, kColSFB = kColSFA + 4 * KSTEPS;
  static constexpr uint32_t kSFBSlot = 4 * KSTEPS;
  static constexpr uint32_t kColEnd = QF ? kColSFB + kSlots * kSFBSlot : kColQ + D / 2;
  static constexpr uint32_t kTmemCols = (kColEnd <= 256) ? 256u : 512u;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kSlots * KTILE;
  static constexpr int kOffKraw = kOffV + kSlots * TILE;
  static constexpr int kOffVraw = kOffKraw + kRawStages * RAW;
  static constexpr int kOffQ4 = kOffVraw + kRawStages * RAW;
  static constexpr int kOffBar = kOffQ4 + QTILE;
  static constexpr int kNumBars = kNumBarriers;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kOffIds = kOffMisc + 64;             // [kMaxIds] block ids
  // the softmax groups' row sums [2 groups][128 rows]
  static constexpr int kOffXchg = kOffIds + kMaxIds * 4;
  static constexpr int kBytes = kOffXchg + 2 * kRows * 4;
  static size_t smem_bytes() {
    const size_t need = (size_t)kBytes + 1024;  // + alignment of the base
    return need > kMinSmem ? need : kMinSmem;
  }
  static_assert(RAW % 16 == 0 && PAGE % 16 == 0, "bulk copies move 16-byte multiples");
  static_assert(TILE % 1024 == 0, "swizzle atoms sit on 1024-byte boundaries");
  static_assert(kColEnd <= 512, "TMEM budget");
  static_assert(!QF || (KTILE % 1024 == 0 && kOffQ4 % 1024 == 0),
                "swizzle atoms sit on 1024-byte boundaries");
  static_assert(kSBufs <= kMaxSBufs && kSlots <= kMaxSlots && kRawStages <= kMaxRawStages,
                "barrier arrays");
  static_assert(kBytes + 1024 <= 227 * 1024, "shared memory per block");
  static_assert(kChunk % BS == 0, "a chunk holds whole pages");
  static_assert(kOffMisc + 64 <= kBytes, "misc block fits");
};

struct Misc {
  uint32_t tmem_base;
  int abort;  // a wait of some role gave up: everyone stops
  uint32_t raw_ok[2][kMaxRawStages];  // per raw stage: bit i = page i of the chunk was copied
};

// Bounded wait that also gives up once another role has aborted the block.
// Waiters share their SM sub-partition's issue slots with the warps doing the
// work they wait for, so they do not spin flat out: kWaitSuspend polls let the
// hardware suspend the thread until the phase completes (or a time hint runs
// out), kWaitSleep polls sleep briefly between tries.
enum WaitMode { kWaitSpin = 0, kWaitSleep = 1, kWaitSuspend = 2 };
constexpr unsigned kRelaxedSleepNs = 64;
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(PREFILL_SUSPEND_NS)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Misc* misc,
                                         uint32_t* status, int mode = kWaitSpin) {
  for (int i = 0; i < kMaxPolls; ++i) {
    if (mode == kWaitSuspend ? mbar_try_wait_suspend(bar, parity) : mbar_try_wait(bar, parity))
      return true;
    if ((i & 127) == 127 && *reinterpret_cast<volatile int*>(&misc->abort)) return false;
    if (mode == kWaitSleep) __nanosleep(kRelaxedSleepNs);
  }
  atomicOr(status, kDevTimeout);
  *reinterpret_cast<volatile int*>(&misc->abort) = 1;
  return false;
}

// Issue the bulk copies of chunk c's pages (K: kv = 0, V: kv = 1) into raw
// stage `st`; pages past kv_end or with a bad block id are not copied (the
// latter flagged). One thread.
template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ void issue_chunk(const AttentionArgs& a, int b, int h, int kv, int c,
                                            int kv_end, uint8_t* raw, uint64_t* bar,
                                            uint32_t* ok_out, uint32_t* status, const int* ids) {
  using S = PrefillShape<D, BS, FMT, QF>;
  const int Hkv = a.num_kv_heads;
  uint32_t ok = 0, bytes = 0;
  long long src[S::PPC];
#pragma unroll
  for (int i = 0; i < S::PPC; ++i) {
    const int p = c * S::PPC + i;
    src[i] = -1;
    if (p * BS < kv_end && p < a.max_blocks_per_seq) {
      const long long blk =
          ids ? ids[p] : __ldg(a.block_table + (long long)b * a.max_blocks_per_seq + p);
      if (blk >= 0 && blk < a.num_blocks) {
        src[i] = ((blk * 2 + kv) * Hkv + h) * (long long)S::PAGE;
        ok |= 1u << i;
        bytes += S::PAGE;
      } else {
        atomicOr(status, kDevBadBlock);
      }
    }
  }
  *ok_out = ok;
  mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
  for (int i = 0; i < S::PPC; ++i)
    if (src[i] >= 0) bulk_g2s(raw + i * S::PAGE, a.cache + src[i], S::PAGE, bar);
}

// Dequantize one chunk from its raw stage into an f16 tile laid out for the
// MMA: 64-column blocks of [64 keys][64 d] f16, 128-byte rows, the 16-byte
// chunk j of row n stored at chunk j ^ (n % 8). A thread converts one scale
// group (16 elements of one key: 8 code bytes and their E4M3 scale) per step:
// warp w, lane l takes keys 8 (w + 4 j) + l % 8 (j = 0, 1) and group l / 8 of
// every 64-column block, so a warp step covers 8 keys x 4 groups and both the
// code loads and the tile stores are free of bank conflicts. Keys at or past
// the visible end, and keys of pages not copied, become zeros. 128 threads.
//
// The thread's offsets are the same for every chunk: computed once.
struct DequantPlan {
  uint32_t row[2];   // byte offset of key j's row in a raw stage
  uint32_t dst[2];   // byte offset of key j's 128-byte row in a tile's first 64-column block
  uint32_t sw0, sw1; // swizzled offsets of the thread's two 16-byte chunks in a row
  uint32_t goff;     // 8 x (group within a 64-column block)
  int n[2];          // the keys, within the chunk
  int pg[2];         // their pages, within the chunk
};

template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ DequantPlan dequant_plan(int gtid) {
  using S = PrefillShape<D, BS, FMT, QF>;
  static_assert(S::kChunk == 64, "the plan covers 64-key chunks with 4 warps");
  const int lane = gtid & 31, gw = gtid >> 5;
  const int n_lo = lane & 7, g_lo = lane >> 3;
  DequantPlan pl;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int n = (gw + 4 * j) * 8 + n_lo;
    pl.n[j] = n;
    pl.pg[j] = n / BS;
    pl.row[j] = (uint32_t)((n / BS) * S::PAGE + (n % BS) * S::F);
    pl.dst[j] = (uint32_t)(n * 128);
  }
  pl.sw0 = (uint32_t)(((2 * g_lo) ^ n_lo) << 4);
  pl.sw1 = (uint32_t)(((2 * g_lo + 1) ^ n_lo) << 4);
  pl.goff = (uint32_t)(8 * g_lo);
  return pl;
}

template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ void dequant_chunk(uint32_t raw, uint32_t ok, uint32_t tile, int lim,
                                              const DequantPlan& pl) {
  using S = PrefillShape<D, BS, FMT, QF>;
  bool valid[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) valid[j] = (pl.n[j] < lim) && ((ok >> pl.pg[j]) & 1u);
#pragma unroll
  for (int dblk = 0; dblk < D / 64; ++dblk) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t row = raw + pl.row[j];
      // (loaded and converted whatever valid says: the stage's bytes exist,
      // stale for a key not copied, and the result is zeroed after)
      uint4 lo, hi;
      {
        if constexpr (FMT) {  // FP8 row: 16 E4M3 bytes -> 16 f16 (exact)
          uint32_t w[4];
          lds_v4(row + 64 * dblk + 2 * pl.goff, w);
          lo.x = e4m3x2_to_f16x2(w[0] & 0xFFFFu);
          lo.y = e4m3x2_to_f16x2(w[0] >> 16);
          lo.z = e4m3x2_to_f16x2(w[1] & 0xFFFFu);
          lo.w = e4m3x2_to_f16x2(w[1] >> 16);
          hi.x = e4m3x2_to_f16x2(w[2] & 0xFFFFu);
          hi.y = e4m3x2_to_f16x2(w[2] >> 16);
          hi.z = e4m3x2_to_f16x2(w[3] & 0xFFFFu);
          hi.w = e4m3x2_to_f16x2(w[3] >> 16);
        } else {  // NVFP4 row: 8 code bytes x one E4M3 scale -> 16 f16 (exact)
          const uint32_t ca = row + 32 * dblk + pl.goff;
          uint32_t c0, c1;
          if constexpr (S::F % 8 == 0) {
            lds_v2(ca, c0, c1);
          } else {
            c0 = ld_shared_u32(ca);
            c1 = ld_shared_u32(ca + 4);
          }
          const uint32_t sb = lds_b8(row + D / 2 + 4 * dblk + (pl.goff >> 3));
          const uint32_t s2 = e4m3x2_to_f16x2(sb * 0x101u);
          uint32_t x[4], y[4];
          e2m1x8_to_f16x2x4(c0, x);
          e2m1x8_to_f16x2x4(c1, y);
          lo = make_uint4(hmul2_u32(x[0], s2), hmul2_u32(x[1], s2), hmul2_u32(x[2], s2),
                          hmul2_u32(x[3], s2));
          hi = make_uint4(hmul2_u32(y[0], s2), hmul2_u32(y[1], s2), hmul2_u32(y[2], s2),
                          hmul2_u32(y[3], s2));
        }
      }
      if (!valid[j]) lo = hi = make_uint4(0u, 0u, 0u, 0u);
      const uint32_t dst = tile + dblk * (S::kChunk * 128) + pl.dst[j];
      sts_v4(dst + pl.sw0, lo);
      sts_v4(dst + pl.sw1, hi);
    }
  }
}

// NVFP4 queries (QF): the K operand of S = Q K^T is the cache's own E2M1 codes
// and E4M3 block scales, so a K chunk is repacked, not converted: each key's
// D/2 code bytes become one 128-byte row of the slot's K-major tile (16-byte
// chunk j stored at j ^ (key % 8)), and the key's 4 scales of K step t (one
// 32-bit word of the raw row) go to byte offset (key % 32) * 16 + (key / 32) * 4
// of the step's 512-byte scale tile: lane key % 32, column key / 32 once copied
// to TMEM (the layout the block-scaled MMA reads its B scale factors in).
// Keys at or past the visible end, and keys of pages not copied, get zero
// codes and scales. 128 threads: thread i takes key i / 2, half i % 2 of its
// row.
template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ void pack_chunk_k(uint32_t raw, uint32_t ok, uint32_t slot, int lim,
                                             int gtid) {
  using S = PrefillShape<D, BS, FMT, QF>;
  const int n = gtid >> 1, hf = gtid & 1;
  const bool valid = (n < lim) && ((ok >> (n / BS)) & 1u);
  const uint32_t row = raw + (n / BS) * S::PAGE + (n % BS) * S::F;
  const uint32_t dst = slot + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
  for (int jj = 0; jj < D / 64; ++jj) {  // this half's 16-byte code chunks
    const int j = hf * (D / 64) + jj;
    uint32_t w[4];
    lds_v4(row + 16 * j, w);
    uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
    if (!valid) v = make_uint4(0u, 0u, 0u, 0u);
    sts_v4(dst + ((j ^ (n & 7)) << 4), v);
  }
#pragma unroll
  for (int tt = 0; tt < S::KSTEPS / 2; ++tt) {  // this half's K steps
    const int t = hf * (S::KSTEPS / 2) + tt;
    uint32_t sw = ld_shared_u32(row + D / 2 + 4 * t);
    if (!valid) sw = 0u;
    sts_u32(slot + S::KCODES + t * 512 + (n & 31) * 16 + (n >> 5) * 4, sw);
  }
}

// Dequantization of one of K (kv = 0) and V (kv = 1), 128 threads: per chunk,
// wait for its raw pages and a free tile slot, convert, and release both.
// Every warp runs at its own pace (no barrier among the four).
template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ void dequant_role(int kv, int nchunk, int kv_end, uint8_t* base,
                                             uint64_t* bars, Misc* misc, uint32_t* status) {
  using S = PrefillShape<D, BS, FMT, QF>;
  const int gtid = threadIdx.x - (kv ? kVGroup0 : kKGroup0);
  const uint32_t raw_s = smem_u32(base + (kv ? S::kOffVraw : S::kOffKraw));
  const uint32_t tiles_s = smem_u32(base + (kv ? S::kOffV : S::kOffK));
  uint64_t* raw_full = bars + (kv ? kBarVraw : kBarKraw);
  uint64_t* raw_empty = bars + kBarRawEmpty + kv * kMaxRawStages;
  uint64_t* full = bars + (kv ? kBarVFull : kBarKFull);
  uint64_t* empty = bars + (kv ? kBarVEmpty : kBarKEmpty);
  const volatile uint32_t* raw_ok = misc->raw_ok[kv];
  const DequantPlan plan = dequant_plan<D, BS, FMT, QF>(gtid);
  for (int c = 0; c < nchunk; ++c) {
    const int st = c % S::kRawStages, slot = c % S::kSlots;
    bool ok = wait_bar(&raw_full[st], (uint32_t)((c / S::kRawStages) & 1), misc, status, KV_WAIT);
    if (ok && c >= S::kSlots)
      ok = wait_bar(&empty[slot], (uint32_t)((c / S::kSlots - 1) & 1), misc, status, KV_WAIT);
    if (!ok) break;  // the block is aborting
    if (QF && kv == 0)
      pack_chunk_k<D, BS, FMT, QF>(raw_s + st * S::RAW, raw_ok[st], tiles_s + slot * S::KTILE,
                                   kv_end - c * S::kChunk, gtid);
    else
      dequant_chunk<D, BS, FMT, QF>(raw_s + st * S::RAW, raw_ok[st], tiles_s + slot * S::TILE,
                                    kv_end - c * S::kChunk, plan);
    // generic-proxy writes of the tile (read by the tensor core) and reads of
    // the raw stage (next written by a bulk copy), both before the arrivals
    fence_proxy_async_smem();
    tc::mbar_arrive(&full[slot]);
    tc::mbar_arrive(&raw_empty[st]);
  }
}

// Page copies of one of K (kv = 0) and V (kv = 1), one thread: chunk c goes
// into raw stage c % kRawStages once every dequant thread has released the
// chunk that stage held. Both copy warps first stage the CTA's block ids in
// shared memory (K and V pages share them). Before exit the thread waits for
// every copy it issued to land (the copies write this CTA's shared memory).
template <int D, int BS, int FMT, bool QF>
__device__ __forceinline__ void copy_role(const AttentionArgs& a, int kv, int b, int h, int nchunk,
                                          int kv_end, uint8_t* base, uint64_t* bars, Misc* misc,
                                          uint32_t* status) {
  using S = PrefillShape<D, BS, FMT, QF>;
  const int lane = threadIdx.x & 31;
  uint8_t* raw = base + (kv ? S::kOffVraw : S::kOffKraw);
  uint64_t* raw_full = bars + (kv ? kBarVraw : kBarKraw);
  uint64_t* raw_empty = bars + kBarRawEmpty + kv * kMaxRawStages;
  uint32_t* raw_ok = misc->raw_ok[kv];
  const int npages = min((kv_end + BS - 1) / BS, a.max_blocks_per_seq);
  int* ids = nullptr;
  if (npages <= kMaxIds) {
    ids = reinterpret_cast<int*>(base + S::kOffIds);
    const int* row = a.block_table + (long long)b * a.max_blocks_per_seq;
    for (int p = kv * 32 + lane; p < npages; p += 64) ids[p] = __ldg(row + p);
    tc::named_sync(kBarCopy, 64);
  }
  if (lane != 0) return;
  int issued = 0;
  for (int c = 0; c < nchunk; ++c) {
    const int st = c % S::kRawStages;
    if (c >= S::kRawStages &&
        !wait_bar(&raw_empty[st], (uint32_t)((c / S::kRawStages - 1) & 1), misc, status,
                  kWaitSleep))
      break;
    issue_chunk<D, BS, FMT, QF>(a, b, h, kv, c, kv_end, raw + st * S::RAW, &raw_full[st], &raw_ok[st],
                            status, ids);
    issued = c + 1;
  }
  // the last copy of each stage (earlier ones were consumed before the stage
  // was refilled) has landed
  for (int k = max(0, issued - S::kRawStages); k < issued; ++k) {
    const int st = k % S::kRawStages;
    for (int i = 0; i < kMaxPolls; ++i)
      if (mbar_try_wait(&raw_full[st], (uint32_t)((k / S::kRawStages) & 1))) break;
  }
}

}  // namespace

// P of one 16-key group of a row: p = exp2(s * qmult - mu) (0 for keys at or
// past glim when MASK), as f16 hi in pw[0..7] (keys in pairs) and
// lo = f16(p - hi) in pw[8..15]; the p are added to ps4.
template <bool MASK>
__device__ __forceinline__ void p_group(const uint32_t (&sv)[16], float qmult, float mu, int glim,
                                        uint32_t (&pw)[16], float (&ps4)[4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float p0 = ex2(fmaf(__uint_as_float(sv[2 * i]), qmult, -mu));
    float p1 = ex2(fmaf(__uint_as_float(sv[2 * i + 1]), qmult, -mu));
    if constexpr (MASK) {
      p0 = (2 * i < glim) ? p0 : 0.0f;
      p1 = (2 * i + 1 < glim) ? p1 : 0.0f;
    }
    ps4[i & 3] += p0 + p1;
    pw[i] = pack_f16x2(p0, p1);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&pw[i]));
    pw[8 + i] = pack_f16x2(p0 - hf.x, p1 - hf.y);
  }
}

// Global scale of an NVFP4 query row with max |q| = amax: the smallest power
// of two g with amax / (6 g) <= 448 (so no block scale saturates), 1 for a
// zero row. With amax in [2^e, 2^(e+1)) and 2688 = 1.3125 * 2^11, that power is
// 2^(e-11) or 2^(e-10).
__device__ __forceinline__ float q_row_global(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  int E;
  frexpf(amax, &E);  // amax in [2^(E-1), 2^E)
  const int k = (E - 1) - 11;
  return (ldexpf(2688.0f, k) >= amax) ? ldexpf(1.0f, k) : ldexpf(1.0f, k + 1);
}

template <int D, int BS, int FMT, bool QF>
__global__ void __launch_bounds__(kThreads, 1) prefill_attention_kernel(const AttentionArgs a) {
  using S = PrefillShape<D, BS, FMT, QF>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kOffBar);
  Misc* misc = reinterpret_cast<Misc*>(base + S::kOffMisc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int Hkv = a.num_kv_heads, G = a.num_q_heads / Hkv;
  const int TQ = kRows / G;  // query tokens per CTA
  const int q_begin = a.qo_indptr[b];
  const int q_len = a.qo_indptr[b + 1] - q_begin;
  if (q_len <= 1) return;  // decode rows are served by the decode kernel
  uint32_t* status = reinterpret_cast<uint32_t*>(a.workspace);
  if (q_len > (int)gridDim.x * TQ && blockIdx.x == 0 && tid == 0)
    atomicOr(status, kDevBadQlen);  // rows beyond the grid are not written
  const int tile_idx = (int)gridDim.x - 1 - (int)blockIdx.x;  // longest (last) tiles first
  const int qtok0 = tile_idx * TQ;
  if (qtok0 >= q_len) return;
  const int L = a.seq_lens[b];
  const int last_tok = min(q_len - 1, qtok0 + TQ - 1);
  const int kv_end = max(0, min(min(L, L - q_len + last_tok + 1), a.max_blocks_per_seq * BS));
  const int nchunk = (kv_end + S::kChunk - 1) / S::kChunk;

  if (tid == 0) {
    for (int i = 0; i < S::kNumBars; ++i) {
      const bool many = (i >= kBarKFull && i < kBarKFull + 2 * kMaxSlots) || i == kBarQReady ||
                        (i >= kBarRawEmpty && i < kBarRawEmpty + 2 * kMaxRawStages);
      const bool pfull = (i >= kBarPFull && i < kBarPFull + 2 * kMaxSBufs) ||
                         (i >= kBarSRead && i < kBarSRead + kMaxSBufs);
      mbar_init(&bars[i], pfull ? 256u : many ? 128u : (i == kBarFin ? 2u : 1u));
    }
    misc->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(&misc->tmem_base, S::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = misc->tmem_base;

  if (warp < 4 || warp >= kSoftmax1Warp0) {
    // ------------------------------------------------ Q, softmax, epilogue:
    // two groups of 128 threads, thread (warp % 4, lane) of each on row
    // r = TMEM lane 32 (warp % 4) + lane; group wg takes keys [wg CH/2,
    // (wg + 1) CH/2) of every chunk and columns [wg D/2, (wg + 1) D/2) of O.
    // Both compute each chunk's max over all its keys and take every decision
    // on the running max from the same values, so they agree on it without
    // exchanging anything; the row sums are added through shared memory at
    // the end.
    const int wg = warp < 4 ? 0 : 1;
    const int r = ((warp & 3) << 5) | lane;
    const int tok = r / G, g = r % G;
    const bool row_ok = (r < TQ * G) && (qtok0 + tok < q_len);
    const int pos = L - q_len + qtok0 + tok;  // absolute position (may be < 0: sees nothing)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float* xsum = reinterpret_cast<float*>(base + S::kOffXchg);  // [2][kRows]
    const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                (long long)(q_begin + qtok0 + tok) * a.q_token_stride +
                                (long long)(h * G + g) * D;
    float mx = 0.0f;
    if (row_ok) {
#pragma unroll 4
      for (int i = 0; i < D / 8; ++i) {
        const uint4 v4 = __ldg(reinterpret_cast<const uint4*>(qrow) + i);
        const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(wv[j] << 16)),
                               fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
      }
    }
    float qmult;
    if constexpr (QF) {
      // NVFP4 queries: the row is quantized with the KV row codec under its
      // global scale g (the smallest power of two with amax / (6 g) <= 448),
      // codes into the Q tile (one 128-byte swizzled row per query row), the
      // 4 scales of K step t into byte (r % 32) * 16 + (r / 32) * 4 of step t's
      // scale tile; g joins the logit scale.
      const float g = q_row_global(mx);
      qmult = a.sm_scale * __ldg(a.kv_scales) * kLog2e * g;
      if (wg == 0) {
        const uint32_t q4 = smem_u32(base + S::kOffQ4);
        const uint32_t qdst = q4 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll 1
        for (int t = 0; t < S::KSTEPS; ++t) {
          uint32_t sw = 0u, cw[8];
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {  // the step's 4 groups of 16
            float x[16];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
              if (row_ok) v4 = __ldg(reinterpret_cast<const uint4*>(qrow + t * 64 + gi * 16) + j);
              const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                x[8 * j + 2 * i] = __uint_as_float(wv[i] << 16);
                x[8 * j + 2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
              }
            }
            const uint32_t sb = quantize_group16(x, g, cw[2 * gi], cw[2 * gi + 1]);
            sw |= sb << (8 * gi);
          }
          // the step's 32 code bytes: 16-byte chunks 2t and 2t + 1 of the row
          sts_v4(qdst + (((2 * t) ^ (r & 7)) << 4), make_uint4(cw[0], cw[1], cw[2], cw[3]));
          sts_v4(qdst + (((2 * t + 1) ^ (r & 7)) << 4), make_uint4(cw[4], cw[5], cw[6], cw[7]));
          sts_u32(q4 + S::QCODES + t * 512 + (r & 31) * 16 + (r >> 5) * 4, sw);
        }
        fence_proxy_async_smem();  // read by the tensor core (MMA, scale copies)
        tc::mbar_arrive(&bars[kBarQReady]);
      }
    } else {
      const int ex = (mx > 0.0f) ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126 : 1;
      const int sh = min(126, max(-126, 15 - ex));
      const float qs = __uint_as_float((uint32_t)(sh + 127) << 23);
      qmult = a.sm_scale * __ldg(a.kv_scales) * kLog2e *
              __uint_as_float((uint32_t)(127 - sh) << 23);
#pragma unroll 1
      for (int blk = 0; wg == 0 && blk < D / 64; ++blk) {  // (group 0 writes Q)
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
          if (row_ok) v4 = __ldg(reinterpret_cast<const uint4*>(qrow + blk * 64) + j);
          const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            w[4 * j + i] = pack_f16x2(__uint_as_float(wv[i] << 16) * qs,
                                      __uint_as_float(wv[i] & 0xFFFF0000u) * qs);
        }
        tc::tmem_st32(tb + lane_off + S::kColQ + blk * 32, w);
      }
      if (wg == 0) {
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&bars[kBarQReady]);
      }
    }

    float m_run = -INFINITY, l_run = 0.0f;
    int done_chunks = 0;
    constexpr int CH = S::kChunk, HC = CH / 2;  // keys per chunk, per group
    static_assert(HC == 32, "a group's half chunk is one 32-column TMEM load");
    for (int c = 0; c < nchunk; ++c) {
      const int sb = c % S::kSBufs;
      const bool ok = wait_bar(&bars[kBarSFull + sb], (uint32_t)((c / S::kSBufs) & 1), misc, status, SM_WAIT);
      if (!__all_sync(0xffffffffu, ok)) break;  // the block is aborting
      tc::fence_after_sync();
      const uint32_t ccol = tb + lane_off + S::kColS + CH * sb;  // the chunk's columns
      const uint32_t scol = ccol + HC * wg;                      // this group's half
      const int limc = min(pos + 1, kv_end) - c * CH;  // keys [c CH, c CH + limc) are visible
      const int lim = limc - HC * wg;                  // the same, from this group's first key
      // pass 1: max of the chunk's visible logits, in log2 units, over all CH
      // keys (both groups compute it: no exchange). When every key of the
      // chunk is visible to every row of the warp (all but the causal edge) and
      // the scale is positive, the max of the raw logits is scaled once
      // (rounding is monotone) and no key is masked.
      const bool unmasked = __all_sync(0xffffffffu, limc >= CH && qmult > 0.0f);
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // (independent chains)
      float cmax;
      if (unmasked) {
#pragma unroll 1
        for (int half = 0; half < CH / 32; ++half) {
          uint32_t sv[32];
          tc::tmem_ld32(ccol + 32 * half, sv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(sv[i]));
        }
        cmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * qmult;
      } else {
#pragma unroll 1
        for (int half = 0; half < CH / 32; ++half) {
          uint32_t sv[32];
          tc::tmem_ld32(ccol + 32 * half, sv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = (32 * half + i < limc) ? __uint_as_float(sv[i]) * qmult : -INFINITY;
            mx4[i & 3] = fmaxf(mx4[i & 3], x);
          }
        }
        cmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      }
      // every logit of the chunk is in registers: the other group may now
      // overwrite its half with P (it waits for this arrival before its first
      // P store; so does this group)
      tc::mbar_arrive(&bars[kBarSRead + sb]);
      // lazy max: move it (and rescale O) only when this chunk exceeds it by > 2^8
      const bool up = (m_run == -INFINITY) ? (cmax > -INFINITY) : (cmax > m_run + kRescaleThresh);
      const bool need_o = up && m_run != -INFINITY;  // O holds earlier contributions
      float alpha = 1.0f;
      if (up) {
        const float m_new = fmaxf(m_run, cmax);
        if (m_run != -INFINITY) alpha = ex2(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      if (__any_sync(0xffffffffu, need_o)) {
        // every PV MMA so far must be done before O is read and rewritten
        // (P-free of chunk c - 1: PV_{c-1} and, in issue order, every PV before it
        // done; that barrier is at most one phase behind here)
        bool wok = wait_bar(&bars[kBarPFree + (c - 1) % S::kSBufs], (uint32_t)(((c - 1) / S::kSBufs) & 1),
                            misc, status);
        if (!__all_sync(0xffffffffu, wok)) break;  // the block is aborting
        {
          tc::fence_after_sync();
#pragma unroll 1
          for (int blk = 0; blk < D / 32; ++blk) {  // the group's half of O
            const uint32_t oc = tb + lane_off + S::kColO + wg * (D / 2) + blk * 16;
            uint32_t o[16];
            tc::tmem_ld16(oc, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tc::tmem_st16(oc, o);
          }
          tc::tmem_wait_st();
        }
      }
      // pass 2: P = exp2(q.k * scale - m) per 16-key group, as f16 hi (8
      // columns, keys in pairs) and lo = f16(P - hi) (the next 8), written over
      // the group's own 16 logit columns (already read)
      const float mu = (m_run == -INFINITY) ? 0.0f : m_run;  // no visible key yet: P = 0
      float ps4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      bool aborted = false;
#pragma unroll 1
      for (int grp = 0; grp < HC / 16; ++grp) {
        uint32_t sv[16], pw[16];
        tc::tmem_ld16(scol + 16 * grp, sv);
        tc::tmem_wait_ld();
        if (unmasked)
          p_group<false>(sv, qmult, mu, 0, pw, ps4);
        else
          p_group<true>(sv, qmult, mu, lim - 16 * grp, pw, ps4);
        // both groups have read this chunk's logits (each reads all of them
        // in pass 1) before either writes P over its half; the first group's
        // P is computed before the wait, so skew between the groups hides
        // behind it
        if (grp == 0 &&
            !__all_sync(0xffffffffu, wait_bar(&bars[kBarSRead + sb], (uint32_t)((c / S::kSBufs) & 1),
                                              misc, status, SM_WAIT))) {
          aborted = true;  // the block is aborting
          break;
        }
        tc::tmem_st16(scol + 16 * grp, pw);
        // group grp of both halves ready: its PV MMAs may start while the
        // next group is computed
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&bars[kBarPFull + 2 * sb + grp]);
      }
      if (aborted) break;
      l_run += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      done_chunks = c + 1;
    }

    // ---- epilogue: o = O / l * v_scale -> fp32 / E4M3 / bf16
    // O is final once every MMA has completed: the one-time barrier the MMA
    // thread commits after its last PV (a per-chunk barrier could still have
    // two chunks outstanding here, which a parity wait cannot tell apart)
    bool have_o = false;
    if (done_chunks == nchunk && nchunk > 0) {
      const bool ok = wait_bar(&bars[kBarFin], 0u, misc, status);
      have_o = __all_sync(0xffffffffu, ok);
    }
    tc::fence_after_sync();
    // the row sum over both groups' keys (the same sum in both: a + b = b + a)
    xsum[wg * kRows + r] = l_run;
    tc::named_sync(kBarSoftmax, 256);
    l_run += xsum[(wg ^ 1) * kRows + r];
    const float v_scale = __ldg(a.kv_scales + 1);
    const float o_scale = __ldg(a.o_scale);
    const float inv_os = 1.0f / o_scale;
    const float scl = (l_run > 0.0f) ? v_scale / l_run : 0.0f;
    const long long obase =
        ((long long)(q_begin + qtok0 + tok) * a.num_q_heads + h * G + g) * D;
    const bool vec8 = (reinterpret_cast<uintptr_t>(a.o_fp8) & 15) == 0;
    const bool vec16 = (reinterpret_cast<uintptr_t>(a.o_bf16) & 15) == 0;
    const bool vec32 = (reinterpret_cast<uintptr_t>(a.o_f32) & 15) == 0;
#pragma unroll 1
    for (int blk = wg * (D / 64); blk < (wg + 1) * (D / 64); ++blk) {  // the group's half of O
      uint32_t o[32];
      if (have_o) {  // (warp-uniform: every lane loads its row)
        tc::tmem_ld32(tb + lane_off + S::kColO + blk * 32, o);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (row_ok) {
      float f[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(o[i]) * scl;
      const long long idx = obase + blk * 32;
      if (a.o_f32) {
        if (vec32) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(a.o_f32 + idx)[i] =
                make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            reinterpret_cast<float2*>(a.o_f32 + idx)[i] = make_float2(f[2 * i], f[2 * i + 1]);
        }
      }
      uint32_t codes[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) codes[i] = f32x2_to_e4m3x2(f[2 * i] * inv_os, f[2 * i + 1] * inv_os);
      if (vec8) {
        uint4* dst = reinterpret_cast<uint4*>(a.o_fp8 + idx);
        dst[0] = make_uint4(codes[0] | codes[1] << 16, codes[2] | codes[3] << 16,
                            codes[4] | codes[5] << 16, codes[6] | codes[7] << 16);
        dst[1] = make_uint4(codes[8] | codes[9] << 16, codes[10] | codes[11] << 16,
                            codes[12] | codes[13] << 16, codes[14] | codes[15] << 16);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          reinterpret_cast<uint16_t*>(a.o_fp8 + idx)[i] = (uint16_t)codes[i];
      }
      if (a.o_bf16) {
        uint32_t bw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t h2 = e4m3x2_to_f16x2(codes[i]);
          const float2 ff = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(ff.x, o_scale), __fmul_rn(ff.y, o_scale));
          bw[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(a.o_bf16) + idx;
        if (vec16) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<uint4*>(ob)[i] = make_uint4(bw[4 * i], bw[4 * i + 1], bw[4 * i + 2], bw[4 * i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) reinterpret_cast<uint32_t*>(ob)[i] = bw[i];
        }
      }
      }  // row_ok
      __syncwarp();
    }
  } else if (warp == kMmaWarp || warp == kSWarp) {
    // ------------------------------------------------ MMA issue: one thread of
    // warp kSWarp issues every S = Q K^T, one thread of warp kMmaWarp every
    // O += P V; each commits its own barriers (a commit tracks the MMAs its
    // thread issued), and the two order through them: S_j is issued once PV_{j-NB}
    // (which read the P buffer S_j overwrites) has completed, PV_c once the
    // softmax has turned S_c into P_c.
    // The whole warp runs the loop (its waits made warp-uniform); one elected
    // lane issues each MMA and commit.
    if (nchunk > 0) {
      constexpr int CH = S::kChunk;
      constexpr int NB = S::kSBufs, NS = S::kSlots;
      auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, wait_bar(bar, parity, misc, status, MMA_WAIT));
      };
      bool ok = true;
      if (warp == kSWarp) {
        constexpr uint32_t kIdescS = tc::idesc_f16(kRows, CH, false);
        constexpr uint32_t kIdescS4 = tc::idesc_mxf4nvf4(kRows, CH);
        const uint32_t kbase = smem_u32(base + S::kOffK);
        const uint32_t q4 = smem_u32(base + S::kOffQ4);
        ok = wait_all(&bars[kBarQReady], 0u);
        if (QF && ok) {
          // Q's scale factors into TMEM once (the copies run before the MMAs
          // this thread issues after them)
          tc::fence_after_sync();
#pragma unroll
          for (int t = 0; t < S::KSTEPS; ++t)
            tc::cp_32x128b_elect(tb + S::kColSFA + 4 * t, tc::plain_desc(q4 + S::QCODES + t * 512));
        }
        for (int j = 0; ok && j < nchunk; ++j) {
          const int sb = j % NB, slot = j % NS;
          ok = wait_all(&bars[kBarKFull + slot], (uint32_t)((j / NS) & 1));
          if (ok && j >= NB) ok = wait_all(&bars[kBarPFree + sb], (uint32_t)((j / NB - 1) & 1));
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t dS = tb + S::kColS + CH * sb;
          if constexpr (QF) {
            // block-scaled S = (Qc SFq)(Kc SFk)^T: K step t reads bytes
            // [32 t, 32 t + 32) of every 128-byte row (start advanced in
            // 16-byte units) and the step's scale columns
            const uint32_t kt = kbase + slot * S::KTILE;
            const uint32_t sfb = tb + S::kColSFB + slot * S::kSFBSlot;
#pragma unroll
            for (int t = 0; t < S::KSTEPS; ++t)
              tc::cp_32x128b_elect(sfb + 4 * t, tc::plain_desc(kt + S::KCODES + t * 512));
            const uint64_t adesc0 = tc::sw128_desc(q4, 16, 1024);
            const uint64_t bdesc0 = tc::sw128_desc(kt, 16, 1024);
#pragma unroll
            for (int t = 0; t < S::KSTEPS; ++t)
              tc::mma_mxf4_elect(dS, adesc0 + (uint64_t)((32 * t) >> 4),
                                 bdesc0 + (uint64_t)((32 * t) >> 4), kIdescS4,
                                 tb + S::kColSFA + 4 * t, sfb + 4 * t, t > 0);
          } else {
            const uint64_t desc0 = tc::sw128_desc(kbase + slot * S::TILE, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // start address advanced in 16-byte units (stays below 2^14 units)
              const uint64_t desc =
                  desc0 + (uint64_t)(((kk >> 2) * (CH * 128) + (kk & 3) * 32) >> 4);
              tc::mma_ts_elect(dS, tb + S::kColQ + kk * 8, desc, kIdescS, kk > 0);
            }
          }
          tc::commit_elect(&bars[kBarKEmpty + slot]);
          tc::commit_elect(&bars[kBarSFull + sb]);
        }
      } else {
        constexpr uint32_t kIdescPV = tc::idesc_f16(kRows, D, true);
        const uint32_t vbase = smem_u32(base + S::kOffV);
        for (int c = 0; ok && c < nchunk; ++c) {
          const int pb = c % NB, slot = c % NS;
          ok = wait_all(&bars[kBarVFull + slot], (uint32_t)((c / NS) & 1));
          const uint64_t desc0 = tc::sw128_desc(vbase + slot * S::TILE, CH * 128, 1024);
          const uint32_t pS = tb + S::kColS + CH * pb;
          // 16-key group g of each half as soon as the softmax has written it:
          // keys 16 g .. and CH/2 + 16 g .. (P hi, then P lo)
#pragma unroll 1
          for (int g = 0; ok && g < CH / 32; ++g) {
            ok = wait_all(&bars[kBarPFull + 2 * pb + g], (uint32_t)((c / NB) & 1));
            if (!ok) break;
            tc::fence_after_sync();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int i = g + hf * (CH / 32);
              const uint64_t desc = desc0 + (uint64_t)((i * 2048) >> 4);
              tc::mma_ts_elect(tb + S::kColO, pS + i * 16, desc, kIdescPV, c > 0 || i > 0);
              tc::mma_ts_elect(tb + S::kColO, pS + i * 16 + 8, desc, kIdescPV, true);
            }
          }
          if (!ok) break;
          tc::commit_elect(&bars[kBarVEmpty + slot]);
          tc::commit_elect(&bars[kBarPFree + pb]);
        }
      }
      // every MMA this warp issued has completed: the final barrier counts
      // both issuers
      tc::commit_elect(&bars[kBarFin]);
      if (warp == kMmaWarp) {
        // (TMEM is released by this warp below, after every MMA has completed)
        for (int i = 0; i < kMaxPolls; ++i)
          if (mbar_try_wait(&bars[kBarFin], 0u)) break;
      }
    }
    __syncwarp();
  } else if (warp == kCopyWarp0 || warp == kCopyWarp0 + 1) {
    copy_role<D, BS, FMT, QF>(a, warp - kCopyWarp0, b, h, nchunk, kv_end, base, bars, misc, status);
  } else {
    // K (warps 5-8) and V (warps 9-12) run one copy of the code
    dequant_role<D, BS, FMT, QF>(tid >= kVGroup0 ? 1 : 0, nchunk, kv_end, base, bars, misc, status);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tb, S::kTmemCols);
  }
}

template <int D, int BS, int FMT, bool QF>
static cudaError_t launch_prefill_t(const AttentionArgs& a, cudaStream_t stream) {
  using S = PrefillShape<D, BS, FMT, QF>;
  const size_t smem = S::smem_bytes();
  auto kern = prefill_attention_kernel<D, BS, FMT, QF>;
  // the attribute is set once per (device, context), under a lock
  static std::mutex attr_mutex;
  static unsigned long long attr_ctx[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  unsigned long long ctx = 0;
  err = current_context_id(&ctx);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(attr_mutex);
    if (ctx == 0 || attr_ctx[dev] != ctx) {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
      attr_ctx[dev] = ctx;
    }
  }
  const int G = a.num_q_heads / a.num_kv_heads;
  const int TQ = kRows / G;
  dim3 grid((a.max_q_len + TQ - 1) / TQ, a.num_kv_heads, a.num_seqs);
  kern<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const AttentionArgs& a, cudaStream_t stream) {
  if (a.flags & kAttnQfp4) {  // NVFP4 queries: head size 256, NVFP4 cache
    if (a.head_size != 256 || a.kv_format != 0) return cudaErrorInvalidValue;
    return a.block_size == 16 ? launch_prefill_t<256, 16, 0, true>(a, stream)
                              : launch_prefill_t<256, 32, 0, true>(a, stream);
  }
#define NVFP4_PREFILL_CASE(DD, BB)                                             \
  if (a.head_size == DD && a.block_size == BB)                                 \
    return a.kv_format ? launch_prefill_t<DD, BB, 1, false>(a, stream)         \
                       : launch_prefill_t<DD, BB, 0, false>(a, stream);
  NVFP4_PREFILL_CASE(64, 16)
  NVFP4_PREFILL_CASE(64, 32)
  NVFP4_PREFILL_CASE(128, 16)
  NVFP4_PREFILL_CASE(128, 32)
  NVFP4_PREFILL_CASE(256, 16)
  NVFP4_PREFILL_CASE(256, 32)
#undef NVFP4_PREFILL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace nvfp4kv
