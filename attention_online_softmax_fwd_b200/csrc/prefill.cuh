// Tiled prefill attention for sm_100a: TMA-staged K/V tiles, tcgen05 MMAs with
// fp32 accumulators in tensor memory, online softmax in registers.
//
// A persistent CTA walks work items (b, hq, 256-row query block), longest
// causal blocks first. The query block is two 128-row tiles, A and B, that
// share every K/V tile the CTA loads. Roles (384 threads, 12 warps):
//   warp 0      TMA producer: Q_A, Q_B once per item, then K_0, K_1, V_0,
//               K_2, V_1, ... into a ring (each K one tile ahead of its V)
//   warps 1, 2  MMA issuers, one thread per query tile; warp 1 owns the TMEM allocation
//   warp 3      idle (it only gives up registers)
//   warps 4-7   softmax of tile A (thread t <-> row t <-> TMEM lane t)
//   warps 8-11  softmax of tile B
// Each of the four SM sub-partitions holds warps w, w + 4, w + 8 (one of warps
// 0-3 and one warp of each softmax warpgroup) and owns a quarter of the
// register file, so the register split is balanced within every sub-partition.
// Tensor memory (512 columns): S_A | S_B | O_A | O_B, fp32.
// Per KV tile j the issuer of tile X issues S_X(j+1) = Q_X K_{j+1}^T as soon as
// the softmax of tile X has copied S_X(j) into registers, and O_X += P_X(j) V_j
// once the softmax has written the bf16 probabilities P_X(j) to shared
// memory; the two tiles' issuers never wait on each other's softmax. So the
// exponentials of tile j overlap the next tile's Q K^T, and the tensor pipe has
// queued work while either softmax warpgroup computes. The two softmax
// warpgroups take turns on the MUFU for their exponentials (the MUFU turns,
// below), so that one group's exponentials overlap the other's score loads and
// P stores.
// The exponentials use a reference maximum that is only raised when the tile
// maximum exceeds it by more than 2^8 (exact: O and l share the reference).
// BLASST tile skip: each softmax warp publishes a vote per 64-key half and the
// MMA issuer combines the four; a warp waits for the others only when its own
// rows would drop the whole tile (then it does no exponentials at all).
#pragma once

#include "common.cuh"

namespace attn {

struct PrefillParams {
  __nv_bfloat16* o;    // [B][S][Hq][D]
  float* lse;          // [B][Hq][S] natural log, or null
  uint8_t* skip_mask;  // [B][Hq][n_qt][n_kt] or null
  int* status;         // caller's device status or null
  int B, S, Hq, Hkv;
  int n_qblocks;       // ceil(S / 256)
  int n_qt, n_kt;      // ceil(S / 128), ceil(S / 64)
  int num_items;       // n_qblocks * B * Hq (< 2^31)
  float scale_log2;    // scale * log2(e)
  float log2_lambda;   // log2(lambda) (tile skip only)
  // chunked prefill over a paged cache (S is then the chunk length Sq)
  const int* block_table;  // [B][max_pages]
  const int* seq_lens;     // [B]: tokens in the cache, the chunk's own included (>= S)
  const __nv_bfloat16* k_pool;   // [num_pages][page_size][Hkv][D]
  const __nv_bfloat16* v_pool;
  int max_pages, num_pages, page_size;
  unsigned long long* skipped_tiles;   // tile skip: count of skipped (query tile, 64-key tile) decisions, or null
  unsigned long long wait_ns;          // pipeline wait limit (kWaitLimitNs unless a test shortens it)
  int withhold_step;                   // test only: the producer leaves out this ring step (-1: none)
};

constexpr int kPfRows = 128;     // rows per query tile
constexpr int kPfKeys = 128;     // keys per K/V tile (two 64-key decision tiles)
constexpr int kPfThreads = 384;
constexpr int kPfProducerWarp = 0, kPfIssuerWarp0 = 1;   // issuer of tile x: warp 1 + x
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Chunked (paged) prefill: up to this many (sequence, query block) pairs are ranked by their
// number of K/V tiles at the start of every CTA, so that the items go out longest first.
constexpr int kPfMaxPairs = 256;
// setmaxnreg split: warps 0-3 drop to kPfRegsLow registers, the softmax warps rise to
// kPfRegsHigh. Per sub-partition: low + 2 * high <= 3 * 168, the launch allocation.
constexpr int kPfRegsLow = 72, kPfRegsHigh = 216;
constexpr int kPfRegPoolNeeded = 128 * kPfRegsLow + 256 * kPfRegsHigh;  // must fit the launch allocation
constexpr int kPfLaunchRegs = 168;   // 168 x 384 = 64512
static_assert(kPfRegsLow + 2 * kPfRegsHigh <= 3 * kPfLaunchRegs, "register split exceeds a sub-partition's share");

template <int D>
struct PrefillSmem {
  static constexpr int kTileBytes = kPfRows * D * 2;            // one Q, K or V tile
  static constexpr int kChunkBytes = kPfRows * 128;             // 64 columns x 128 rows, SW128
  static constexpr int kPBytes = kPfRows * kPfKeys * 2;         // one P tile (bf16)
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kQ = 0;                                  // Q_A, Q_B
  static constexpr int kP = 2 * kTileBytes;                     // P_A, P_B
  static constexpr int kRing = kP + 2 * kPBytes;
  static constexpr int kBars = kRing + kStages * kTileBytes;
  // barrier indices (pairs are per query tile)
  static constexpr int bQFull = 0, bQEmpty = 2, bSFull = 4, bSFree = 6, bPFull = 8, bPVDone = 10, bOEmpty = 12,
                       bTeardown = 14, bTurn = 15, bKVFull = 17,
                       bKVEmpty = 17 + kStages, kNumBars = 17 + 2 * kStages;
  static constexpr int kMisc = kBars + 8 * kNumBars;            // tmem base, flags
  static constexpr int kVotes = (kMisc + 16 + 15) / 16 * 16;    // skip votes [2][4][4] ints
  static constexpr int kOrder = kMisc + 256;                    // paged: item costs and their order (below)
  static constexpr int kTotal = kOrder + kPfMaxPairs * 6;
  static_assert(kVotes + 128 <= kOrder, "skip votes exceed the misc area");
  static constexpr int kDynamic = kTotal + 1024;
  static_assert(kDynamic <= 232448, "shared memory per block");
};

// TMEM columns: S_A | S_B | O_A | O_B
__device__ __forceinline__ uint32_t pf_col_s(int x) { return uint32_t(x) * 128u; }
template <int D>
__device__ __forceinline__ uint32_t pf_col_o(int x) { return 256u + uint32_t(x) * D; }

// S = Q K^T: D/16 MMAs of 128 x 128 x 16; the K-major descriptors advance 32 B
// within a 128-byte swizzle row and one 16 KB chunk per 64 columns.
template <int D>
__device__ __forceinline__ void pf_issue_qk(uint32_t d_tmem, uint64_t qdesc, uint64_t kdesc) {
  constexpr uint32_t idesc = make_idesc_bf16(128, kPfKeys, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off16 = uint64_t(((kk / 4) * (kPfRows * 128) + (kk % 4) * 32) >> 4);
    umma_ss(d_tmem, qdesc + off16, kdesc + off16, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V: P K-major (keys contiguous) and V MN-major, both from shared
// memory; 8 MMAs of 128 x D x 16 keys. 16 keys = 32 B of a P row and 2 KB of V.
// Bit h of skip_halves leaves out the four MMAs of 64-key half h.
template <int D>
__device__ __forceinline__ void pf_issue_pv(uint32_t d_tmem, uint64_t pdesc, uint64_t vdesc, bool accumulate,
                                            int skip_halves) {
  constexpr uint32_t idesc = make_idesc_bf16(128, D, 0, 1);
  bool acc = accumulate;
#pragma unroll
  for (int kk = 0; kk < kPfKeys / 16; ++kk) {
    if ((skip_halves >> (kk / 4)) & 1) continue;
    const uint64_t poff16 = uint64_t(((kk / 4) * (kPfRows * 128) + (kk % 4) * 32) >> 4);
    umma_ss(d_tmem, pdesc + poff16, vdesc + uint64_t((kk * 16 * 128) >> 4), idesc, acc ? 1u : 0u);
    acc = true;
  }
}

// Tile-wide skip decision of one query tile and one K/V tile: the AND of the
// four softmax warps' votes (bit h set: every row of the warp lets 64-key half h
// go). A vote word is (tag << 2) | bits, the tag naming the tile in the
// warpgroup's sequence, so a stale word is never taken for a fresh one. The
// four words of a tile are adjacent and 16-byte aligned.
__device__ __forceinline__ int4 pf_votes_v4(const volatile int* words) {
  int4 w;
  asm volatile("ld.volatile.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
               : "r"(smem_u32(const_cast<const int*>(words)))
               : "memory");
  return w;
}
__device__ __forceinline__ bool pf_votes_all_in(const int4& w, int tag) {
  return ((w.x >> 2) == tag) & ((w.y >> 2) == tag) & ((w.z >> 2) == tag) & ((w.w >> 2) == tag);
}

// Waits (bounded by the pipeline wait limit) for all four votes; -1 on timeout.
// Kept out of line: it runs only when a vote is late, and inlined it would
// crowd the registers of the softmax loop.
__device__ __forceinline__ int pf_tile_decision_wait(const volatile int* words, int tag, volatile int* abort_flag,
                                                  int* user_status, unsigned long long limit_ns) {
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    const int4 w = pf_votes_v4(words);
    if (pf_votes_all_in(w, tag)) return w.x & w.y & w.z & w.w & 3;
    if ((i & 31u) == 0) {
      if (*abort_flag) return -1;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        raise_status(user_status, ATTN_ERR_TIMEOUT);
        return -1;
      }
    }
  }
}

__device__ __forceinline__ int pf_tile_decision(const volatile int* words, int tag, volatile int* abort_flag,
                                                int* user_status, unsigned long long limit_ns) {
  const int4 w = pf_votes_v4(words);
  if (pf_votes_all_in(w, tag)) return w.x & w.y & w.z & w.w & 3;
  return pf_tile_decision_wait(words, tag, abort_flag, user_status, limit_ns);
}

// The V load of a K/V tile shared by the two query tiles: the halves that both
// drop (bit h: 64-key half h), once both warpgroups' votes are in; -1 on
// timeout. tag_x is the tile's vote sequence number in warpgroup x, 0 when query
// tile x does not visit the tile (it then drops both halves).
__device__ __forceinline__ int pf_dropped_by_both(const volatile int* votes, int tag0, int tag1,
                                                  volatile int* abort_flag, int* user_status,
                                                  unsigned long long limit_ns) {
  unsigned long long t0 = 0;
  for (uint32_t i = 0;; ++i) {
    int d = 3;
    bool in = true;
    if (tag0) {
      const int4 w = pf_votes_v4(votes + (tag0 & 3) * 4);
      in = in && pf_votes_all_in(w, tag0);
      d &= w.x & w.y & w.z & w.w;
    }
    if (tag1) {
      const int4 w = pf_votes_v4(votes + 16 + (tag1 & 3) * 4);
      in = in && pf_votes_all_in(w, tag1);
      d &= w.x & w.y & w.z & w.w;
    }
    if (in) return d & 3;
    // the votes come once the softmax warps have the tile's row maxima, often a few hundred
    // cycles away: sleep between polls, so that this warp takes no issue slots from the
    // softmax warps that share its SM sub-partition
    __nanosleep(64);
    if (i == 0) {
      t0 = global_timer_ns();
    } else if ((i & 31u) == 0) {
      if (*abort_flag) return -1;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        raise_status(user_status, ATTN_ERR_TIMEOUT);
        return -1;
      }
    }
  }
}

// The order of one item's K and V tiles in the ring: K_0 .. K_{L-1}, then V_j and
// K_{j+L} in turn, then the last V tiles. With L = 2 each K_{j+1} is loaded just
// before V_j. (A larger L would let every skip decision arrive before its V is
// due, but with three ring slots it leaves V_j waiting for the slot of K_{j+1}
// and exposes the V latency on every tile: 1.5x the dense time when nothing is
// skipped.)
template <int L>
__device__ __forceinline__ void pf_ring_step(int step, int n, bool& is_k, int& tile) {
  const int a = n < L ? n : L;
  if (step < a) { is_k = true; tile = step; return; }
  const int st = step - a, m = n - a;
  if (st < 2 * m) {
    is_k = (st & 1) != 0;
    tile = (st >> 1) + (is_k ? L : 0);
    return;
  }
  is_k = false;
  tile = m + (st - 2 * m);
}

// MUFU turns. The two query tiles' softmax warpgroups share the
// SM sub-partitions (warps w and w + 4 on each), and left to themselves they run in step:
// both wait on the MUFU for their exponentials at once, then both leave it idle while
// they load scores and store P. So on the K/V tiles that both query tiles visit they
// take turns, passed with a pair of mbarriers of four arrivals: tile A's exponentials of
// tile j follow tile B's of tile j - 1, and tile B's follow tile A's of tile j, so that
// one group's exponentials overlap the other's non-MUFU work. The turn is handed on
// after the first kTurnHandoff of the 64 exponential pairs: one warp alone keeps its
// sub-partition's MUFU only about two-thirds busy, so the next group's first
// exponentials fill it while this group issues its last quarter (measured best among
// hand-overs after 32 to 64 pairs). With the tile skip, a group that drops a whole tile
// takes the turn and hands it on at once, so that both groups count the same tiles.

constexpr int kTurnHandoff = 48;

// Row-sum pairs (exact, as rounded for P V), added and scaled without contraction.
__device__ __forceinline__ float2 sum2_add(float2 a, float2 b) {
  return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
}
__device__ __forceinline__ float2 sum2_scale(float2 a, float s) {
  return make_float2(__fmul_rn(a.x, s), __fmul_rn(a.y, s));
}
// The sums of the 64-key halves that decision d keeps (bit h: half h skipped).
__device__ __forceinline__ float2 sum2_kept(const float2 (&h)[2], int d) {
  const float2 a = (d & 1) ? make_float2(0.f, 0.f) : h[0];
  const float2 b = (d & 2) ? make_float2(0.f, 0.f) : h[1];
  return make_float2(a.x + b.x, a.y + b.y);
}

// This thread's row of S from tensor memory (128 columns), with keys past the
// causal diagonal or the sequence end set to -inf.
template <bool CAUSAL>
__device__ __forceinline__ void pf_load_scores(uint32_t taddr, float (&s)[kPfKeys], int key0, int row, int row0,
                                               int S) {
  uint32_t sr[kPfKeys];
  ATTN_TMEM_LD32_NOWAIT(taddr + 0, sr + 0);
  ATTN_TMEM_LD32_NOWAIT(taddr + 32, sr + 32);
  ATTN_TMEM_LD32_NOWAIT(taddr + 64, sr + 64);
  ATTN_TMEM_LD32_NOWAIT(taddr + 96, sr + 96);
  tmem_ld_wait();
  ATTN_REG_FENCE32(sr + 0);
  ATTN_REG_FENCE32(sr + 32);
  ATTN_REG_FENCE32(sr + 64);
  ATTN_REG_FENCE32(sr + 96);
#pragma unroll
  for (int e = 0; e < kPfKeys; ++e) s[e] = __uint_as_float(sr[e]);
  const float neg_inf = -__int_as_float(0x7f800000);
  const bool full_tile = (!CAUSAL || key0 + kPfKeys - 1 <= row0) && (key0 + kPfKeys <= S);
  if (!full_tile) {
#pragma unroll
    for (int e = 0; e < kPfKeys; ++e) {
      const int key = key0 + e;
      if ((CAUSAL && key > row) || key >= S) s[e] = neg_inf;
    }
  }
}

// Zero source for the paged loads of key slots past a sequence's end.
__device__ __align__(16) uint8_t g_pf_zero16[16];

// Group g (16 keys) of a K or V tile of 128 keys gathered from the page pool
// (chunked prefill): page sizes are multiples of 16, so a group never
// straddles two pages; the eight groups of a tile complete on `bar` for
// kTileBytes in all. A group wholly past
// the sequence end, or in a page the block table does not hold (reported as
// ATTN_ERR_DEVICE_BOUNDS), is filled with zeros by an out-of-range page
// coordinate, which reads nothing. The group holding the sequence end is
// copied 16 bytes at a time into the swizzled positions, zeros past the end,
// so no slot past the end is read: those slots may hold anything, and a NaN
// there would survive a zero probability in P V.
// The raw block-table entry of group g of K/V tile t of sequence b, or
// num_pages (nothing to read) for a group past the sequence end.
__device__ __forceinline__ int pf_page_entry(const PrefillParams& p, int b, int t, int g, int n_keys) {
  const int key = t * kPfKeys + g * 16;
  const int lp = key / p.page_size;
  return (key < n_keys && lp < p.max_pages) ? __ldg(&p.block_table[size_t(b) * p.max_pages + lp]) : p.num_pages;
}

template <int D>
__device__ __forceinline__ void pf_load_paged_group(uint8_t* dst, const CUtensorMap* tm16,
                                                    const __nv_bfloat16* pool, uint64_t* bar,
                                                    const PrefillParams& p, int kvh, int key0, int n_keys, int g,
                                                    int entry) {
  const int key = key0 + g * 16;
  const int slot0 = key % p.page_size;
  int phys = p.num_pages;   // out of range: zeros
  if (key < n_keys) {
    if (entry >= 0 && entry < p.num_pages) phys = entry;
    else raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
  }
  if (key + 16 <= n_keys || phys == p.num_pages) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_4d(dst + c * (kPfRows * 128) + g * 16 * 128, tm16, bar, c * 64, kvh, slot0, phys);
  } else {
    for (int r = 0; r < 16; ++r) {
      const int row = g * 16 + r;
      const bool valid = key + r < n_keys;
      const uint8_t* src_row =
          reinterpret_cast<const uint8_t*>(pool + ((size_t(phys) * p.page_size + slot0 + r) * p.Hkv + kvh) * D);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          bulk_load(dst + c * (kPfRows * 128) + row * 128 + ((u ^ (row & 7)) << 4),
                    valid ? src_row + c * 128 + u * 16 : g_pf_zero16, 16, bar);
    }
  }
}

// Record the decisions for K/V tile jt (two 64-key tiles) of query tile qt:
// 1 skipped, 0 kept; tiles past the causal diagonal or the sequence stay untouched.
template <bool CAUSAL>
__device__ __forceinline__ void pf_write_skip_mask(const PrefillParams& p, int b, int hq, int qt, int jt,
                                                   int last_row, int decision) {
  uint8_t* mrow = p.skip_mask + ((size_t(b) * p.Hq + hq) * p.n_qt + qt) * p.n_kt;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k64 = jt * kPfKeys + h * 64;
    const bool visited = k64 < p.S && (!CAUSAL || k64 <= last_row);
    if (visited) mrow[k64 / 64] = uint8_t((decision >> h) & 1);
  }
}

// The visited 64-key tiles among the two of K/V tile jt that decision d drops.
template <bool CAUSAL>
__device__ __forceinline__ int pf_count_skipped(const PrefillParams& p, int jt, int last_row, int decision) {
  int n = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k64 = jt * kPfKeys + h * 64;
    const bool visited = k64 < p.S && (!CAUSAL || k64 <= last_row);
    n += (visited && ((decision >> h) & 1)) ? 1 : 0;
  }
  return n;
}

// PAGED: chunked prefill. Query row i of sequence b sits at position
// L_b - S + i (L_b = seq_lens[b]) and sees cached keys 0 .. L_b - S + i; the K
// and V tiles are gathered from the page pool through the block table, one
// box of 16 keys at a time (pf_load_paged_tile; tm_k / tm_v then map the pools as
// {D, Hkv, page_size, P} with 16-slot boxes).
// SKIP: tm_vh maps V with boxes of 64 rows (one 64-key half of a tile), so that
// the producer loads only the halves that one of the two query tiles keeps.
// DBG (the test entry point only): the producer's and issuers' wait limit comes
// from p.wait_ns and the producer leaves out ring step p.withhold_step; every
// other instantiation waits up to kWaitLimitNs and withholds nothing.
template <int D, bool CAUSAL, bool SKIP, bool PAGED = false, bool DBG = false>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_vh,
                   const PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NS = L::kStages;
  constexpr int kTmemCols = 512;
  constexpr int kLead = 2;   // K tiles loaded before the first V (pf_ring_step)
  const unsigned long long wait_lim = DBG ? p.wait_ns : kWaitLimitNs;


  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  // skip votes [tile x][sequence slot, 4][softmax warp, 4]; slot = tile sequence number mod 4
  volatile int* votes = reinterpret_cast<volatile int*>(smem + L::kVotes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 32; ++i) votes[i] = 0;   // tag 0 never names a tile
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars[L::bQFull + x], 1);
      mbar_init(&bars[L::bQEmpty + x], 1);
      mbar_init(&bars[L::bSFull + x], 1);
      mbar_init(&bars[L::bSFree + x], 4);    // one arrival per softmax warp
      mbar_init(&bars[L::bPFull + x], 4);
      mbar_init(&bars[L::bPVDone + x], 1);
      mbar_init(&bars[L::bOEmpty + x], 4);
    }
    mbar_init(&bars[L::bTeardown], 2);
    mbar_init(&bars[L::bTurn + 0], 4);   // tile A may take its exponentials (one arrival per tile-B warp)
    mbar_init(&bars[L::bTurn + 1], 4);   // tile B may take its exponentials (one arrival per tile-A warp)
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars[L::bKVFull + s], 1);
      mbar_init(&bars[L::bKVEmpty + s], 2);   // both MMA issuers release each slot
    }
    fence_mbar_init();
  }
  if (warp == kPfIssuerWarp0) {
    tmem_alloc(tmem_base_smem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  // The CTA's items: round r takes item r * grid + b, with the CTA order b
  // reversed on odd rounds (a snake), so that the CTAs that take the longer
  // item of one round take the shorter of the next: with items in decreasing
  // length, every CTA ends within about one tile of the others. In the chunked
  // (paged) prefill an item's length also depends on its sequence's cached
  // prefix, so its items are put in that order first (ranked below); beyond
  // kPfMaxPairs pairs they keep the (query block, sequence) order and the plain
  // stride, since the snake over an unsorted order pairs long items with long
  // ones (measured 15 % slower).
  // The chunked (paged) prefill ranks its (sequence, query block) pairs by their K/V tile
  // count, in shared memory, so that its items also go out longest first (pf_rank_pairs below).
  const int n_pairs = p.B * p.n_qblocks;
  const bool ranked = PAGED && n_pairs <= kPfMaxPairs;
  const uint16_t* pair_order = reinterpret_cast<const uint16_t*>(smem + L::kOrder + kPfMaxPairs * 4);
  auto pf_item_of = [&](int round) {
    const int b = ((!PAGED || ranked) && (round & 1)) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x);
    return round * int(gridDim.x) + b;
  };
  // Item decode shared by all roles: longest causal blocks first; the G query
  // heads of one KV head are adjacent so their K/V tiles are reused from L2.
  auto item_coords = [&](int item, int& qb, int& b, int& hq) {
    if (ranked) {
      const int pair = pair_order[item / p.Hq];
      b = pair / p.n_qblocks;
      qb = pair % p.n_qblocks;
      hq = item % p.Hq;
      return;
    }
    const int per = p.B * p.Hq;
    qb = p.n_qblocks - 1 - item / per;
    const int rem = item % per;
    b = rem / p.Hq;
    hq = rem % p.Hq;
  };
  auto tile_rows = [&](int qb, int x) { return max(0, min(kPfRows, p.S - qb * 2 * kPfRows - x * kPfRows)); };
  // PAGED: position of query row 0 of sequence b (its cache length minus the
  // chunk length); a length outside [S, capacity] is clamped and, when asked,
  // reported as ATTN_ERR_DEVICE_BOUNDS
  auto seq_offset = [&](int b, bool report) {
    if constexpr (!PAGED) {
      return 0;
    } else {
      const int cap = p.max_pages * p.page_size;
      int len = __ldg(&p.seq_lens[b]);
      if (len < p.S || len > cap) {
        if (report) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
        len = max(p.S, min(len, cap));
      }
      return len - p.S;
    }
  };
  auto tile_nkv = [&](int qb, int x, int rows, int off) {
    if (rows == 0) return 0;
    if (CAUSAL) return (off + qb * 2 * kPfRows + x * kPfRows + rows - 1) / kPfKeys + 1;
    return (p.S + kPfKeys - 1) / kPfKeys;
  };

  if (ranked) {
    // Rank the pairs by K/V tiles (both query tiles' counts), most first, ties in pair order:
    // with the items in that order the snake gives every CTA about the same work, whatever the
    // sequences' cached prefixes. Every CTA computes the same order.
    uint32_t* cost = reinterpret_cast<uint32_t*>(smem + L::kOrder);
    uint16_t* order = reinterpret_cast<uint16_t*>(smem + L::kOrder + kPfMaxPairs * 4);
    for (int i = int(threadIdx.x); i < n_pairs; i += int(blockDim.x)) {
      const int b = i / p.n_qblocks, qb = i % p.n_qblocks;
      const int off = seq_offset(b, false);
      cost[i] = uint32_t(tile_nkv(qb, 0, tile_rows(qb, 0), off) + tile_nkv(qb, 1, tile_rows(qb, 1), off));
    }
    __syncthreads();
    for (int i = int(threadIdx.x); i < n_pairs; i += int(blockDim.x)) {
      const uint32_t c = cost[i];
      int rank = 0;
      for (int j = 0; j < n_pairs; ++j) {
        const uint32_t cj = cost[j];
        rank += (cj > c || (cj == c && j < i)) ? 1 : 0;
      }
      order[rank] = uint16_t(i);
    }
    __syncthreads();
  }

  // Register split: warps 0-3 give up registers, the softmax warpgroups take them
  // (kPfRegPoolNeeded is checked against the launch allocation on the host).
  if (warp < 4) {
    setmaxnreg_dec<kPfRegsLow>();
    if (warp == kPfProducerWarp && PAGED) {
      // ============================================================ TMA producer (paged)
      // Lane 0 waits for free slots and arms the barriers; lanes 0-7 each copy
      // one 16-key group of a tile, so the block-table loads and the copies of a
      // tile are issued in parallel.
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int slot = 0;
      uint32_t phase = 0;
      uint32_t qe_bits = 3u;
      uint32_t pend_mask = 0, pend_ph = 0;
      bool ok = true;
      for (int round = 0, item = pf_item_of(0); item < p.num_items && ok; item = pf_item_of(++round)) {
        int qb, b, hq;
        item_coords(item, qb, b, hq);
        const int kvh = hq / (p.Hq / p.Hkv);
        const int off = seq_offset(b, false);
        const int rows0 = tile_rows(qb, 0), rows1 = tile_rows(qb, 1);
        const int n = max(tile_nkv(qb, 0, rows0, off), tile_nkv(qb, 1, rows1, off));
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if ((x == 0 ? rows0 : rows1) == 0 || !ok) continue;
          int w = 1;
          if (lane == 0)
            w = mbar_wait(&bars[L::bQEmpty + x], (qe_bits >> x) & 1u, abort_flag, p.status, wait_lim) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; continue; }
          qe_bits ^= 1u << x;
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars[L::bQFull + x], L::kTileBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + L::kQ + x * L::kTileBytes + c * L::kChunkBytes, &tm_q, &bars[L::bQFull + x],
                          c * 64, qb * 2 * kPfRows + x * kPfRows, hq, b);
          }
        }
        // Block-table entries: this lane's group of the next K tile is fetched
        // one K tile ahead; V_t reuses the entry of K_t.
        const int n_keys = off + p.S;
        const int g = lane & 7;
        int pre = pf_page_entry(p, b, 0, g, n_keys);
        int entry_even = p.num_pages, entry_odd = p.num_pages;   // of the last K tiles with even / odd index
        for (int step = 0; step < 2 * n && ok; ++step) {
          bool is_k;
          int tile;
          pf_ring_step<kLead>(step, n, is_k, tile);
          const int key0 = tile * kPfKeys;
          if (is_k) {
            if (tile & 1) entry_odd = pre; else entry_even = pre;
            pre = pf_page_entry(p, b, tile + 1, g, n_keys);
          }
          const int entry = (tile & 1) ? entry_odd : entry_even;
          int w = 1;
          if (lane == 0) w = mbar_wait(&bars[L::bKVEmpty + slot], phase ^ 1u, abort_flag, p.status, wait_lim) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
          if (lane == 0) mbar_arrive_expect_tx(&bars[L::bKVFull + slot], L::kTileBytes);
          if (lane < kPfKeys / 16)
            pf_load_paged_group<D>(smem + L::kRing + slot * L::kTileBytes, is_k ? &tm_k : &tm_v,
                                   is_k ? p.k_pool : p.v_pool, &bars[L::bKVFull + slot], p, kvh, key0, n_keys,
                                   lane, entry);
          pend_mask |= 1u << slot;
          pend_ph = (pend_ph & ~(1u << slot)) | (phase << slot);
          if (++slot == NS) { slot = 0; phase ^= 1u; }
        }
      }
      if (!ok && lane == 0) {
        for (int s = 0; s < NS; ++s)
          if (pend_mask & (1u << s)) mbar_drain(&bars[L::bKVFull + s], (pend_ph >> s) & 1u);
      }
      __syncwarp();
    } else if (warp == kPfProducerWarp) {
      // ============================================================ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t qe_bits = 3u;
        uint32_t pend_mask = 0, pend_ph = 0;
        int vseq[2] = {0, 0};   // SKIP: the tiles each softmax warpgroup has voted on (its vote sequence)
        bool prev_dropped = false;          // SKIP: both query tiles dropped the whole previous V tile
        int pend_tag0 = 0, pend_tag1 = 0;   // SKIP: votes of a V tile loaded without its decision
        int gstep = 0;          // ring steps of this CTA (for the test-only withheld step)
        bool ok = true;
        for (int round = 0, item = pf_item_of(0); item < p.num_items && ok; item = pf_item_of(++round)) {
          int qb, b, hq;
          item_coords(item, qb, b, hq);
          const int kvh = hq / (p.Hq / p.Hkv);
          const int off = seq_offset(b, false);
          const int rows0 = tile_rows(qb, 0), rows1 = tile_rows(qb, 1);
          const int nkv0 = tile_nkv(qb, 0, rows0, off), nkv1 = tile_nkv(qb, 1, rows1, off);
          const int n = max(nkv0, nkv1);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if ((x == 0 ? rows0 : rows1) == 0 || !ok) continue;
            if (!mbar_wait(&bars[L::bQEmpty + x], (qe_bits >> x) & 1u, abort_flag, p.status, wait_lim)) {
              ok = false;
              continue;
            }
            qe_bits ^= 1u << x;
            mbar_arrive_expect_tx(&bars[L::bQFull + x], L::kTileBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + L::kQ + x * L::kTileBytes + c * L::kChunkBytes, &tm_q, &bars[L::bQFull + x],
                          c * 64, qb * 2 * kPfRows + x * kPfRows, hq, b);
          }
          // the order in which the MMA issuers consume the tiles (pf_ring_step)
          for (int step = 0; step < 2 * n && ok; ++step) {
            bool is_k;
            int tile;
            pf_ring_step<kLead>(step, n, is_k, tile);
            const int key0 = tile * kPfKeys;
            int halves = 3;   // bit h: 64-key half h of the tile is loaded
            if constexpr (SKIP) {
              if (!is_k) {
                // V_tile is due before the softmax warps have voted on it. After a tile that both
                // query tiles dropped, the producer waits for the votes and loads only the halves
                // that one of the two keeps, so a run of dropped tiles reads no V; after a kept
                // tile it loads the whole tile at once, which keeps the dense pipeline.
                const int tag0 = tile < nkv0 ? ++vseq[0] : 0;   // 0: this query tile does not visit it
                const int tag1 = tile < nkv1 ? ++vseq[1] : 0;
                if (tile == 0) {
                  prev_dropped = false;   // a unit's first tile is never dropped
                } else if (pend_tag0 | pend_tag1) {
                  // the previous tile's votes (loaded at once): cast right after its scores were read,
                  // normally in by the time the ring has a slot for this V tile
                  const int d = pf_dropped_by_both(votes, pend_tag0, pend_tag1, abort_flag, p.status, wait_lim);
                  if (d < 0) { ok = false; break; }
                  prev_dropped = d == 3;
                }
                pend_tag0 = pend_tag1 = 0;
                if (prev_dropped) {
                  const int dropped = pf_dropped_by_both(votes, tag0, tag1, abort_flag, p.status, wait_lim);
                  if (dropped < 0) { ok = false; break; }
                  halves = ~dropped & 3;
                  prev_dropped = dropped == 3;
                } else {
                  pend_tag0 = tag0;   // loaded without waiting; its votes are read at the next V
                  pend_tag1 = tag1;
                }
              }
            }
            if (!mbar_wait(&bars[L::bKVEmpty + slot], phase ^ 1u, abort_flag, p.status, wait_lim)) {
              ok = false;
              break;
            }
            if (!DBG || gstep++ != p.withhold_step) {
              uint8_t* dst = smem + L::kRing + slot * L::kTileBytes;
              if (halves == 3) {
                mbar_arrive_expect_tx(&bars[L::bKVFull + slot], L::kTileBytes);
                const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                  tma_load_4d(dst + c * L::kChunkBytes, tm, &bars[L::bKVFull + slot], c * 64, key0, kvh, b);
              } else {
                mbar_arrive_expect_tx(&bars[L::bKVFull + slot], uint32_t(__popc(halves)) * (L::kTileBytes / 2));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  if (!((halves >> h) & 1)) continue;
#pragma unroll
                  for (int c = 0; c < D / 64; ++c)
                    tma_load_4d(dst + c * L::kChunkBytes + h * (L::kChunkBytes / 2), &tm_vh, &bars[L::bKVFull + slot],
                                c * 64, key0 + 64 * h, kvh, b);
                }
              }
              pend_mask |= 1u << slot;
              pend_ph = (pend_ph & ~(1u << slot)) | (phase << slot);
            }
            if (++slot == NS) { slot = 0; phase ^= 1u; }
          }
        }
        if (!ok) {
          for (int s = 0; s < NS; ++s)
            if (pend_mask & (1u << s)) mbar_drain(&bars[L::bKVFull + s], (pend_ph >> s) & 1u);
        }
      }
    } else if (warp == kPfIssuerWarp0 || warp == kPfIssuerWarp0 + 1) {
      // ============================================================ MMA issuers
      // One thread per query tile x (warp 1: A, warp 2: B). Both walk the whole
      // K/V ring of every item and arrive on each slot's empty barrier (count 2),
      // whether or not their tile uses the slot; an issuer never runs more than
      // one ring phase ahead because it waits for each slot's load first.
      if (lane == 0) {
        const int x = warp - kPfIssuerWarp0;
        const uint32_t q_desc_addr = smem_u32(smem + L::kQ + x * L::kTileBytes);
        const uint32_t p_desc_addr = smem_u32(smem + L::kP + x * L::kPBytes);
        const uint32_t ring_addr = smem_u32(smem + L::kRing);
        const uint32_t d_s = tmem + pf_col_s(x), d_o = tmem + pf_col_o<D>(x);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t qf_ph = 0u, sfree_ph = 0u, pf_ph = 0u, oe_ph = 1u;
        bool qk_started = false;  // a Q K^T has been issued for this tile in this kernel
        int seq = 0;              // P V tiles of this query tile so far (skip-vote sequence)
        bool ok = true;

        for (int round = 0, item = pf_item_of(0); item < p.num_items && ok; item = pf_item_of(++round)) {
          int qb, b, hq;
          item_coords(item, qb, b, hq);
          const int off = seq_offset(b, false);
          const int rows0 = tile_rows(qb, 0), rows1 = tile_rows(qb, 1);
          const int n = max(tile_nkv(qb, 0, rows0, off), tile_nkv(qb, 1, rows1, off));
          const int nkv = tile_nkv(qb, x, x == 0 ? rows0 : rows1, off);
          if (nkv > 0) {
            if (!mbar_wait(&bars[L::bQFull + x], qf_ph, abort_flag, p.status, wait_lim)) break;
            qf_ph ^= 1u;
          }
          bool pv_started = false;  // a P V product was issued for this tile in this item
          // ring uses of the item, in the producer's order (pf_ring_step)
          for (int step = 0; step < 2 * n && ok; ++step) {
            bool is_k;
            int tile;
            pf_ring_step<kLead>(step, n, is_k, tile);
            const int cur = slot;
            const uint32_t cph = phase;
            if (++slot == NS) { slot = 0; phase ^= 1u; }
            if (!mbar_wait(&bars[L::bKVFull + cur], cph, abort_flag, p.status, wait_lim)) { ok = false; break; }
            tc_fence_after();
            if (is_k && tile < nkv) {
              // S_x(tile) = Q_x K_tile^T, once the softmax has copied out S_x(tile - 1)
              if (qk_started) {
                if (!mbar_wait(&bars[L::bSFree + x], sfree_ph, abort_flag, p.status, wait_lim)) { ok = false; break; }
                sfree_ph ^= 1u;
                tc_fence_after();
              }
              qk_started = true;
              pf_issue_qk<D>(d_s, make_sdesc_sw128(q_desc_addr, 16, 1024),
                             make_sdesc_sw128(ring_addr + cur * L::kTileBytes, 16, 1024));
              umma_commit(&bars[L::bSFull + x]);
              if (tile + 1 == nkv) umma_commit(&bars[L::bQEmpty + x]);   // last Q K^T of this tile
            } else if (!is_k && tile < nkv) {
              // O_x += P_x(tile) V_tile
              if (!mbar_wait(&bars[L::bPFull + x], pf_ph, abort_flag, p.status, wait_lim)) { ok = false; break; }
              pf_ph ^= 1u;
              tc_fence_after();
              int skip_halves = 0;
              if constexpr (SKIP) {
                // every softmax warp voted before arriving on P_full
                ++seq;
                skip_halves = pf_tile_decision(votes + x * 16 + (seq & 3) * 4, seq, abort_flag, p.status, wait_lim);
                if (skip_halves < 0) { ok = false; break; }
              }
              if (skip_halves != 3) {
                if (!pv_started) {
                  // first P V of this item: the previous item's epilogue must have read O_x
                  if (!mbar_wait(&bars[L::bOEmpty + x], oe_ph, abort_flag, p.status, wait_lim)) { ok = false; break; }
                  oe_ph ^= 1u;
                  tc_fence_after();
                }
                pf_issue_pv<D>(d_o, make_sdesc_sw128(p_desc_addr, 16, 1024),
                               make_sdesc_sw128(ring_addr + cur * L::kTileBytes, L::kChunkBytes, 1024), pv_started,
                               skip_halves);
                pv_started = true;
              }
              umma_commit(&bars[L::bPVDone + x]);   // P_x free; after the last tile: O_x final
            }
            umma_commit(&bars[L::bKVEmpty + cur]);
          }
        }
        // every MMA this thread issued must finish before the TMEM is released
        umma_commit(&bars[L::bTeardown]);
        mbar_drain(&bars[L::bTeardown], 0);
      }
    }
  } else {
    setmaxnreg_inc<kPfRegsHigh>();
    // ============================================================ softmax warpgroups
    const int x = (warp - 4) / 4;          // 0: tile A, 1: tile B
    const int wq = warp & 3;               // TMEM lane quadrant
    const int t = wq * 32 + lane;          // row within the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t taddr_s = tmem + lane_off + pf_col_s(x);
    const uint32_t taddr_o = tmem + lane_off + pf_col_o<D>(x);
    // this thread's row of P (K-major, 128-byte swizzle, two 64-key chunks)
    uint8_t* prow = smem + L::kP + x * L::kPBytes + t * 128;
    const float neg_inf = -__int_as_float(0x7f800000);
    // The softmax waits stop on their own limit only (the full one: the test entry point shortens the
    // producer's and issuers' waits, which then give up first; these follow within the full limit).
    int own_timeout_only = 0;
    volatile int* no_abort = reinterpret_cast<volatile int*>(&own_timeout_only);
    uint32_t sf_ph = 0, pvd_ph = 0;
    uint32_t turn_ph = 0;         // MUFU turns waited for (parity)
    bool turn_started = false;    // this warp has taken a turn (tile A waits from its second on)
    int seq = 0;   // K/V tiles of this query tile so far (skip-vote sequence)
    bool ok = true;

    for (int round = 0, item = pf_item_of(0); item < p.num_items && ok; item = pf_item_of(++round)) {
      int qb, b, hq;
      item_coords(item, qb, b, hq);
      const int off = seq_offset(b, x == 0 && t == 0);
      const int n_keys = PAGED ? off + p.S : p.S;   // keys in the cache (the sequence)
      const int rows = tile_rows(qb, x);
      const int nkv = tile_nkv(qb, x, rows, off);
      if (nkv == 0) continue;
      // K/V tiles that both query tiles of the block visit (they alternate on the MUFU there)
      const int n_common = min(nkv, tile_nkv(qb, 1 - x, tile_rows(qb, 1 - x), off));
      const int row0 = qb * 2 * kPfRows + x * kPfRows;
      const int row = row0 + t;
      const bool row_valid = t < rows;
      const int last_row = row0 + rows - 1;
      float m_ref = neg_inf, m_true = neg_inf;
      int n_skipped = 0;   // SKIP, thread 0: dropped visited 64-key tiles of this query tile
      // Row sums at the reference m_ref: .x sums the probabilities (-> LSE); .y
      // normalises O and differs from .x by the bf16 rounding of each half's largest
      // probability: under the lagging reference a dominant key has P up to 2^8, and
      // its rounding, left out of the sum, would scale the whole output row.
      float2 l = make_float2(0.f, 0.f);

      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&bars[L::bSFull + x], sf_ph, no_abort, p.status)) { ok = false; break; }
        sf_ph ^= 1u;
        tc_fence_after();
        const int key0 = j * kPfKeys;
        float s[kPfKeys];
        pf_load_scores<CAUSAL>(taddr_s, s, key0, off + row, off + row0, n_keys);
        // S_x is in registers: the tensor pipe may overwrite it with the next tile
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::bSFree + x]);
        // row maxima of the two 64-key halves (raw scores; scale > 0 commutes with max)
        float mx[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int bb = h * 64;
          float a0 = max3f(s[bb + 0], s[bb + 1], s[bb + 2]), a1 = max3f(s[bb + 3], s[bb + 4], s[bb + 5]);
          float a2 = max3f(s[bb + 6], s[bb + 7], s[bb + 8]), a3 = max3f(s[bb + 9], s[bb + 10], s[bb + 11]);
#pragma unroll
          for (int e = 12; e < 60; e += 8) {
            a0 = max3f(a0, s[bb + e + 0], s[bb + e + 1]);
            a1 = max3f(a1, s[bb + e + 2], s[bb + e + 3]);
            a2 = max3f(a2, s[bb + e + 4], s[bb + e + 5]);
            a3 = max3f(a3, s[bb + e + 6], s[bb + e + 7]);
          }
          a0 = max3f(a0, s[bb + 60], s[bb + 61]);
          a1 = max3f(a1, s[bb + 62], s[bb + 63]);
          mx[h] = fmaxf(max3f(a0, a1, a2), a3);
        }
        float r2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) r2[h] = (mx[h] == neg_inf) ? neg_inf : mx[h] * p.scale_log2;

        // Tile skip (SKIP only): this warp's vote, bit h set when every one of its
        // rows lets 64-key half h go. The running maximum used by the test takes
        // in every visited score: a half that is skipped lies below it by
        // -log2(lambda) > 0, so this equals the maximum over kept halves.
        // A warp that keeps a half does not wait for the other votes: it computes
        // the exponentials at once. That is exact whatever the outcome, since a
        // skipped half can neither raise the reference maximum (it lies below the
        // running maximum, which is within 2^8 of the reference) nor set it when
        // it is raised. The issuer leaves skipped halves out of P V, and the row
        // sums of the kept halves are added to l once P is handed over.
        // A warp that would drop the whole tile waits for the tile-wide decision
        // with its scores still in registers (S_x was released at once, as in the
        // dense kernel, so the next Q K^T is not held back by the vote).
        int vote = 0, decision = -1;
        bool skip_all = false;
        if constexpr (SKIP) {
          const float lam2 = p.log2_lambda;
          const bool ok0 = !row_valid || r2[0] == neg_inf || (m_true != neg_inf && r2[0] - m_true < lam2);
          const float m1 = fmaxf(m_true, r2[0]);
          const bool ok1 = !row_valid || r2[1] == neg_inf || (m1 != neg_inf && r2[1] - m1 < lam2);
          m_true = fmaxf(m1, r2[1]);
          vote = (__all_sync(0xffffffffu, ok0) ? 1 : 0) | (__all_sync(0xffffffffu, ok1) ? 2 : 0);
          ++seq;
          if (lane == 0) votes[x * 16 + (seq & 3) * 4 + wq] = (seq << 2) | vote;
          if (vote == 3) {
            decision = pf_tile_decision(votes + x * 16 + (seq & 3) * 4, seq, no_abort, p.status, kWaitLimitNs);
            if (decision < 0) { ok = false; break; }
            skip_all = decision == 3;
          }
          if (skip_all) {
            // the whole tile is dropped: no exponentials, no P, no P V (l, O and
            // the reference stay as they are); keep the P V phase count and the
            // MUFU turns in step (the turn is taken and handed on at once)
            if (j < n_common) {
              if (x == 1 || turn_started) {
                if (!mbar_wait(&bars[L::bTurn + x], turn_ph, no_abort, p.status)) { ok = false; break; }
                turn_ph ^= 1u;
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars[L::bTurn + 1 - x]);
              turn_started = true;
            }
            if (j > 0) {
              if (!mbar_wait(&bars[L::bPVDone + x], pvd_ph, no_abort, p.status)) { ok = false; break; }
              pvd_ph ^= 1u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[L::bPFull + x]);
            if (p.skip_mask && t == 0) pf_write_skip_mask<CAUSAL>(p, b, hq, qb * 2 + x, j, last_row, 3);
            if (t == 0) n_skipped += pf_count_skipped<CAUSAL>(p, j, last_row, 3);
            continue;
          }
        }
        uint32_t pk[kPfKeys / 2];   // this row's probabilities, bf16 pairs
        float alpha = 1.f;
        bool raise = false;
        float2 hsum[2];   // the halves' row sums
        {
          const float m_tile = fmaxf(r2[0], r2[1]);
          // raise the reference maximum only when needed (or on the first finite tile)
          raise = (m_tile != neg_inf) && (m_ref == neg_inf || m_tile > m_ref + kRescaleThreshold);
          if (raise) {
            alpha = (m_ref == neg_inf) ? 0.f : fast_exp2(m_ref - m_tile);
            m_ref = m_tile;
          }
          float offset = (m_ref == neg_inf) ? 0.f : m_ref;
          {
            // MUFU turn: on the tiles both query tiles visit, tile A takes its exponentials
            // after tile B's of the previous such tile, and tile B after tile A's of the same one
            if (j < n_common && (x == 1 || turn_started)) {
              if (!mbar_wait(&bars[L::bTurn + x], turn_ph, no_abort, p.status)) { ok = false; break; }
              turn_ph ^= 1u;
            }
            asm volatile("" : "+f"(offset) : : "memory");   // no exponential before the turn
          }
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t negoff2 = f2_pack(-offset, -offset);
          uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int e = 0; e < kPfKeys / 2; ++e) {
            const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), scale2, negoff2);
            float x0, x1;
            f2_unpack(xx, x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            pk[e] = pack_bf16x2(p0, p1);
            sum2[(e / 32) * 2 + (e & 1)] = f2_add(sum2[(e / 32) * 2 + (e & 1)], f2_pack(p0, p1));
            {
              if (e == kTurnHandoff - 1 && j < n_common) {
                // the first kTurnHandoff pairs are issued (their results are in registers)
#pragma unroll
                for (int u = 0; u < kTurnHandoff; ++u) asm volatile("" : "+r"(pk[u]) : : "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[L::bTurn + 1 - x]);
                turn_started = true;
              }
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float sa, sb, sc, sd;
            f2_unpack(sum2[2 * h], sa, sb);
            f2_unpack(sum2[2 * h + 1], sc, sd);
            hsum[h].x = (sa + sb) + (sc + sd);
            // The normalising sum takes the largest probability of the half as
            // rounded for P V (the same fma and exp2 as in the loop above give the
            // same value): that term dominates the rounding error of the weights
            // (P up to 2^8 under the lagging reference), the others average out.
            const float pm = fast_exp2(fmaf(mx[h], p.scale_log2, -offset));
            hsum[h].y = (mx[h] == neg_inf) ? hsum[h].x : hsum[h].x + (bf16_lo(pack_bf16x2(pm, pm)) - pm);
          }
          if constexpr (!SKIP) {
            // all exponentials are in registers here (the schedule the hand-over point was chosen with)
            ATTN_REG_FENCE32(pk);
            ATTN_REG_FENCE32(pk + 32);
            asm volatile("" : "+f"(hsum[0].y), "+f"(hsum[1].y) : : "memory");
          }
        }
        // P_x(j-1) must have been consumed (and O_x updated) before P_x(j) is written
        // and before any rescale of O_x; the exponentials above overlapped that P V.
        if (j > 0) {
          if (!mbar_wait(&bars[L::bPVDone + x], pvd_ph, no_abort, p.status)) { ok = false; break; }
          pvd_ph ^= 1u;
          tc_fence_after();
        }
        // l <- l * alpha + (kept halves' sums), without contraction so that lambda = 0
        // through the skip path rounds exactly like the dense path
        l = sum2_scale(l, alpha);
        if constexpr (!SKIP) l = sum2_add(l, sum2_kept(hsum, 0));
        {
          if (__any_sync(0xffffffffu, raise && j > 0)) {
            // rescale this warp's rows of O (every P V of earlier tiles has completed)
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              ATTN_TMEM_LD32(taddr_o + c * 32, r);
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              ATTN_TMEM_ST32(taddr_o + c * 32, r);
            }
            tmem_st_wait();
          }
          // P row: 16-byte units of 8 keys; 128-byte swizzle puts unit u at (u mod 8) ^ (row mod 8)
#pragma unroll
          for (int u = 0; u < kPfKeys / 8; ++u) {
            const int chunk = u >> 3, uu = u & 7;
            *reinterpret_cast<uint4*>(prow + chunk * L::kChunkBytes + ((uu ^ (t & 7)) << 4)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
          fence_proxy_async_smem();   // the tensor pipe reads P through the async proxy
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::bPFull + x]);
        if constexpr (SKIP) {
          // The other warps voted before their exponentials, so by now the
          // decision is normally complete; fold in the sums of the kept halves.
          const int d = decision >= 0 ? decision
                                      : pf_tile_decision(votes + x * 16 + (seq & 3) * 4, seq, no_abort, p.status,
                                                         kWaitLimitNs);
          if (d < 0) { ok = false; break; }
          l = sum2_add(l, sum2_kept(hsum, d));
          if (p.skip_mask && t == 0) pf_write_skip_mask<CAUSAL>(p, b, hq, qb * 2 + x, j, last_row, d);
          if (t == 0) n_skipped += pf_count_skipped<CAUSAL>(p, j, last_row, d);
        }
      }
      if (!ok) break;

      if (SKIP && t == 0 && n_skipped && p.skipped_tiles) atomicAdd(p.skipped_tiles, (unsigned long long)n_skipped);

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait(&bars[L::bPVDone + x], pvd_ph, no_abort, p.status)) { ok = false; break; }
      pvd_ph ^= 1u;
      tc_fence_after();
      const float inv_l = (l.y > 0.f) ? 1.f / l.y : 0.f;
      __nv_bfloat16* orow = p.o + ((size_t(b) * p.S + row) * p.Hq + hq) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        ATTN_TMEM_LD32(taddr_o + c * 32, r);
        if (row_valid) {
          uint4 w[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wp[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = w[e];
        }
      }
      if (row_valid && p.lse)
        p.lse[(size_t(b) * p.Hq + hq) * p.S + row] =
            (l.x > 0.f) ? (m_ref + __log2f(l.x)) * 0.69314718055994531f : neg_inf;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bOEmpty + x]);
    }
  }

  __syncwarp();  // reconverge the producer and MMA warps (one lane worked)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPfIssuerWarp0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
