// Paged single-token decode: split-KV attention kernel + log-sum-exp merge.
//
// Work item = (sequence, split, KV head). A persistent CTA walks its items in
// a strided order. One producer warp streams the item's 64-token tiles of K
// and V from the page pool into a shared-memory ring with TMA, one copy per
// (page chunk, K|V), addressed through the block table. The page pool is seen
// as 5-D {64 columns, D/64 column blocks, head, slot, page} so that one copy
// moves a chunk's whole head dimension; it lands as rows of 128 bytes
// (token-major, column block minor) with the 128-byte swizzle, which keeps the
// consumers' ldmatrix reads to at most two-way bank conflicts. The producer reads the next item's length and first
// block-table window while it streams the current item, and ships each item's
// query rows (one bulk copy) and metadata with its first tile, so neither side
// waits on a dependent global load when an item starts.
//
// Four consumer warps each take 16 tokens of a tile. The G query heads that
// share the KV head are the rows of a 16-row operand (rows >= G are zero), so
// q.K^T and P.V are two small matrix products per tile, done with
// mma.m16n8k16 (bf16 in, fp32 accumulate, in registers). The online softmax
// (running reference maximum, sum, accumulator) runs per warp in the
// accumulator registers; the four warps' states are merged in a fixed order
// at the end of the item. With the tile skip enabled, the warps exchange
// their tile maxima once per tile (one named barrier) so that every warp sees
// the tile's true row maxima and the unit's true running maximum.
// A split's result is written as a partial (O / l, log2-sum-exp); the merge
// kernel combines the splits of a sequence. A sequence with one split is
// written directly by the split kernel.
#pragma once

#include "common.cuh"

namespace attn {

struct DecodeParams {
  const __nv_bfloat16* q;      // [N][Hq][D]
  const int32_t* block_table;  // [N][max_pages]
  const int32_t* seq_lens;     // [N]
  __nv_bfloat16* o;            // [N][Hq][D]
  float* lse;                  // [N][Hq] (natural log) or null
  float* ws_o;                 // [N][max_splits][Hq][D] fp32 partial outputs (normalised)
  float* ws_lse;               // [N][max_splits][Hq] fp32 partial log2-sum-exp
  uint8_t* skip_mask;          // [N][Hkv][max_tiles] (per_head: [N][Hq][max_tiles]) or null
  int* status;                 // caller's device status word or null
  int num_seqs, Hq, Hkv, page_size, max_pages, num_pages;
  int split_tokens, max_splits, max_tiles;
  int chunk;          // tokens per TMA copy: min(page_size, 64)
  float scale_log2;   // softmax scale * log2(e)
  float log2_lambda;  // log2(lambda) for the tile skip
  float v_scale;      // FP8 cache: V = v_scale * code (the K scale is folded into scale_log2)
  int per_head;       // tile skip decided for each query head alone, not for the KV head's group
  long long num_items;
  int static_items;   // head-group kernel: at most one item per CTA, item = blockIdx.x (no ticket counter)
  // two-pass tile-skip decode (decode_blasst.cuh); the work items are chunks of
  // chunk_tokens tokens (a divisor of split_tokens), the decision units are splits
  float* ws_s;        // scaled scores (log2 units) [N][Hkv / HG][tok64][HG][G]
  float* ws_tmax;     // row maxima of every 64-token tile [N][Hq][max_tiles]
  float* ws_cmax;     // row maxima of every chunk [N][Hq][max_chunks]
  float* ws_cpre;     // splits of more than 16 chunks: running maximum at every chunk start [N][Hq][max_chunks],
                      // else null
  unsigned long long* skipped_tiles;   // count of skipped decisions, or null
  int chunk_tokens, max_chunks, tok64;   // pass 1's work item (chunk maxima per chunk)
  int chunk2_tokens, max_chunks2;        // pass 2's work item (a multiple of chunk_tokens, one partial each)
};

constexpr int kDecTile = 64;          // tokens per tile (= BLASST decision tile)
constexpr int kDecConsumerWarps = 4;  // 16 tokens of each tile per warp
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr float kDecRescaleThreshold = 8.0f;  // log2 units

// What the producer tells the consumers about a stage.
struct TileInfo {
  int seq, split, kvh, t0;
  int ntok;   // valid tokens of the tile from t0
  int bad;    // bit c: page chunk c was outside the pool (not loaded)
  int flags;  // bit 0: first tile of the item (its query rows are in the stage), bit 1: last tile,
              // bit 2: no tile, this CTA's work is done
  int len;    // sequence length (clamped to the block table's capacity)
};

template <int D, int G>
struct DecodeSmem {
  static constexpr int kTileBytes = kDecTile * D * 2;          // one K or V tile
  static constexpr int kQBytes = G * D * 2;                    // the item's query rows
  static constexpr int kStageBytes = (2 * kTileBytes + kQBytes + 1023) / 1024 * 1024;  // K, V, q
  // as many stages (at most 6 for D = 128, 11 for D = 64) as fit beside the combine buffers
  static constexpr int kFixed = 16 * 12 + 4 * 2 * kDecConsumerWarps * 16 + 8 * kDecConsumerWarps * G +
                                4 * kDecConsumerWarps * G * D + 1024 + 64;
  static constexpr int kFit = (232448 - kFixed) / (kStageBytes + 48);
  static constexpr int kStages = (D == 128 ? 6 : 11) < kFit ? (D == 128 ? 6 : 11) : kFit;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kFull = kRing;                                   // mbarriers
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kInfo = kEmpty + 8 * kStages;                    // TileInfo per stage
  static constexpr int kRed = kInfo + 32 * kStages;                     // [2][warps][16] floats
  static constexpr int kCombM = kRed + 4 * 2 * kDecConsumerWarps * 16;  // [warps][G] floats
  static constexpr int kCombL = kCombM + 4 * kDecConsumerWarps * G;     // [warps][G] floats
  static constexpr int kCombO = (kCombL + 4 * kDecConsumerWarps * G + 15) / 16 * 16;  // [warps][G][D]
  static constexpr int kTotal = kCombO + 4 * kDecConsumerWarps * G * D;
  static constexpr int kDynamic = kTotal + 1024;                        // slack for alignment
  static_assert(kDynamic <= 232448, "shared memory per block");
  static_assert(kStages >= 2, "ring depth");
};

__device__ __forceinline__ void decode_item_coords(long long item, int Hkv, int max_splits, int& seq, int& split,
                                                   int& kvh) {
  kvh = int(item % Hkv);
  long long rest = item / Hkv;
  split = int(rest % max_splits);
  seq = int(rest / max_splits);
}

// Byte offset of 16-byte chunk `c` (0 .. D/8-1) of token `r` in a swizzled K or V
// tile: 128-byte row (r * D/64 + c / 8), unit (c mod 8) XOR (row mod 8).
template <int D>
__device__ __forceinline__ uint32_t swz_off(int r, int c) {
  const int row = r * (D / 64) + (c >> 3);
  return uint32_t(row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

template <int D, int G, bool SKIP>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p) {
  static_assert(G >= 1 && G <= 16, "query heads per KV head");
  using L = DecodeSmem<D, G>;
  launch_dependents();   // let the merge kernel be scheduled early; it waits for this grid to finish
  constexpr int NS = L::kStages;
  constexpr int KS = D / 16;   // k-steps of q.K^T
  constexpr int NT = D / 8;    // 8-column tiles of O

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + L::kInfo);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* comb_m = reinterpret_cast<float*>(smem + L::kCombM);
  float* comb_l = reinterpret_cast<float*>(smem + L::kCombL);
  float* comb_o = reinterpret_cast<float*>(smem + L::kCombO);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const int nchunks = kDecTile / p.chunk;
    const uint32_t chunk_bytes = uint32_t(p.chunk) * D * 2;   // one K (or V) chunk, both halves
    int slot = 0;
    uint32_t phase = 0;
    uint32_t pending = 0;  // stages with copies issued, for the abort path
    uint32_t pending_phase = 0;
    bool ok = true;
    // The next candidate item's length and first block-table window are loaded
    // one item ahead; the window does not depend on the length (entries past
    // the sequence end are read but never used).
    int nx_len = 0, nx_win = -1;
    {
      const long long it = blockIdx.x;
      if (it < p.num_items) {
        int sq, sp, kh;
        decode_item_coords(it, p.Hkv, p.max_splits, sq, sp, kh);
        nx_len = __ldg(&p.seq_lens[sq]);
        const int e = (((sp * p.split_tokens) / p.page_size) & ~31) + lane;
        nx_win = e < p.max_pages ? __ldg(&p.block_table[size_t(sq) * p.max_pages + e]) : -1;
      }
    }
    for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      int seq, split, kvh;
      decode_item_coords(item, p.Hkv, p.max_splits, seq, split, kvh);
      int len = nx_len;
      int win_cur = nx_win;
      {
        const long long it = item + gridDim.x;
        if (it < p.num_items) {
          int sq, sp, kh;
          decode_item_coords(it, p.Hkv, p.max_splits, sq, sp, kh);
          nx_len = __ldg(&p.seq_lens[sq]);
          const int e = (((sp * p.split_tokens) / p.page_size) & ~31) + lane;
          nx_win = e < p.max_pages ? __ldg(&p.block_table[size_t(sq) * p.max_pages + e]) : -1;
        }
      }
      if (len > capacity || len < 0) {
        if (lane == 0 && split == 0 && kvh == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
        len = len < 0 ? 0 : capacity;
      }
      const int t_begin = split * p.split_tokens;
      if (t_begin >= len) continue;
      const int t_end = min(t_begin + p.split_tokens, len);
      const int32_t* bt_row = p.block_table + size_t(seq) * p.max_pages;
      int win = (t_begin / p.page_size) >> 5;
      int win_next;
      {
        const int e = (win + 1) * 32 + lane;
        win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
      }
      const __nv_bfloat16* qsrc = p.q + (size_t(seq) * p.Hq + size_t(kvh) * G) * D;
      for (int t0 = t_begin; t0 < t_end; t0 += kDecTile) {
        const int e0 = t0 / p.page_size;  // first entry of this tile; a tile never straddles a window
        if ((e0 >> 5) != win) {
          win = e0 >> 5;
          win_cur = win_next;
          const int e = (win + 1) * 32 + lane;
          win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
        }
        if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        const int p0 = t0 + lane * p.chunk;
        const int mine =
            __shfl_sync(0xffffffffu, win_cur, (e0 & 31) + (lane < nchunks ? lane * p.chunk / p.page_size : 0));
        int page = -1, in_page = 0;
        bool valid = false, bad = false;
        if (lane < nchunks && p0 < len) {
          page = mine;
          in_page = p0 % p.page_size;
          valid = page >= 0 && page < p.num_pages;
          bad = !valid;
        }
        const uint32_t valid_mask = __ballot_sync(0xffffffffu, valid);
        const uint32_t bad_mask = __ballot_sync(0xffffffffu, bad);
        const bool first = t0 == t_begin;
        uint8_t* stage = smem + slot * L::kStageBytes;
        if (lane == 0) {
          if (bad_mask) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
          TileInfo ti;
          ti.seq = seq; ti.split = split; ti.kvh = kvh; ti.t0 = t0;
          ti.ntok = min(kDecTile, len - t0);
          ti.bad = int(bad_mask);
          ti.flags = (first ? 1 : 0) | (t0 + kDecTile >= t_end ? 2 : 0);
          ti.len = len;
          info[slot] = ti;
          mbar_arrive_expect_tx(&full[slot], __popc(valid_mask) * chunk_bytes * 2 + (first ? uint32_t(L::kQBytes) : 0u));
          if (first) bulk_load(stage + 2 * L::kTileBytes, qsrc, uint32_t(L::kQBytes), &full[slot]);
        }
        __syncwarp();
        if (valid) {
          uint8_t* kbase = stage;
          uint8_t* vbase = stage + L::kTileBytes;
          const uint32_t off = uint32_t(lane) * chunk_bytes;   // the chunk's first token row
          tma_load_5d(kbase + off, &tm_k, &full[slot], 0, 0, kvh, in_page, page);
          tma_load_5d(vbase + off, &tm_v, &full[slot], 0, 0, kvh, in_page, page);
        }
        pending |= 1u << slot;
        pending_phase = (pending_phase & ~(1u << slot)) | (phase << slot);
        if (++slot == NS) { slot = 0; phase ^= 1u; }
      }
    }
    if (ok && mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) {
      // end-of-work marker: a stage with no copies
      if (lane == 0) {
        TileInfo ti{};
        ti.flags = 4;
        info[slot] = ti;
        mbar_arrive_expect_tx(&full[slot], 0u);
      }
      __syncwarp();
    } else {
      ok = false;
    }
    if (!ok && lane == 0) {
      for (int s = 0; s < NS; ++s)
        if (pending & (1u << s)) mbar_drain(&full[s], (pending_phase >> s) & 1u);
    }
  } else {
    // ------------------------------------------------------------ consumer warps
    const float neg_inf = -__int_as_float(0x7f800000);
    const int g = lane >> 2;         // accumulator row (query head within the group)
    const int tq = lane & 3;         // column pair within an 8-column tile
    const bool row0_valid = g < G;   // rows g and g + 8
    const bool row1_valid = g + 8 < G;
    int slot = 0;
    uint32_t phase = 0;
    int red_par = 0;
    int no_abort = 0;  // consumers stop only on their own timeout (see mbar_wait)
    bool ok = true;
    const uint32_t ring_addr = smem_u32(smem);

    // The consumers follow the stages the producer fills, until a stage marked
    // as the end of this CTA's work.
    int seq = 0, split = 0, kvh = 0, n_splits = 0;
    uint32_t qa[KS][4];
    float o[NT][4];
    float m_ref[2] = {neg_inf, neg_inf};   // per-warp exponent reference, rows g and g + 8
    float m_true[2] = {neg_inf, neg_inf};  // unit's running max of kept tiles (tile skip)
    float l_part[2] = {0.f, 0.f};          // this lane's share of the row sums (-> LSE)
    float lr_part[2] = {0.f, 0.f};         // the same as rounded to bf16 for P V (-> normalises O)

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) {
        ok = false;
        break;
      }
      const TileInfo ti = info[slot];
      if (ti.flags & 4) break;   // end of work
      const int ntok = ti.ntok;
      const uint32_t bad = uint32_t(ti.bad);
      const int t0 = ti.t0;
      if (ti.flags & 1) {
        // first tile of an item: its query rows (A operand, rows >= G zero) came with this stage
        seq = ti.seq; split = ti.split; kvh = ti.kvh;
        n_splits = (ti.len + p.split_tokens - 1) / p.split_tokens;
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(smem + slot * L::kStageBytes + 2 * L::kTileBytes);
        const int h0 = row0_valid ? g : 0, h1 = row1_valid ? g + 8 : 0;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qa[ks][0] = row0_valid ? qs[h0 * (D / 2) + ks * 8 + tq] : 0u;
          qa[ks][1] = row1_valid ? qs[h1 * (D / 2) + ks * 8 + tq] : 0u;
          qa[ks][2] = row0_valid ? qs[h0 * (D / 2) + ks * 8 + 4 + tq] : 0u;
          qa[ks][3] = row1_valid ? qs[h1 * (D / 2) + ks * 8 + 4 + tq] : 0u;
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m_ref[0] = m_ref[1] = neg_inf;
        m_true[0] = m_true[1] = neg_inf;
        l_part[0] = l_part[1] = 0.f;
        lr_part[0] = lr_part[1] = 0.f;
      }
      const bool last_tile = (ti.flags & 2) != 0;
      const uint32_t kaddr = ring_addr + slot * L::kStageBytes;
      const uint32_t vaddr = kaddr + L::kTileBytes;
      const int tok_base = warp * 16;

      // ---- S = q K^T for this warp's 16 tokens (two 8-token column tiles); the
      // k-steps alternate between two accumulators per column tile so that
      // consecutive MMAs do not wait on each other
      float s[2][4];
      {
        float sp[2][2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int a = 0; a < 2; ++a) sp[j][a][0] = sp[j][a][1] = sp[j][a][2] = sp[j][a][3] = 0.f;
        const int mi = lane >> 3, r = lane & 7;
        const int tok = tok_base + (mi >> 1) * 8 + r;
        uint32_t b[KS][4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) ldsm_x4(kaddr + swz_off<D>(tok, ks * 2 + (mi & 1)), b[ks][0], b[ks][1], b[ks][2], b[ks][3]);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          mma_bf16_16816(sp[0][ks & 1], qa[ks], b[ks][0], b[ks][1]);
          mma_bf16_16816(sp[1][ks & 1], qa[ks], b[ks][2], b[ks][3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[j][e] = sp[j][0][e] + sp[j][1][e];
      }
      // ---- scale to log2 units and mask tokens past the end or in invalid pages
      const bool tile_clean = (ntok == kDecTile) && (bad == 0);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = tok_base + j * 8 + 2 * tq + (e & 1);
          float v = s[j][e] * p.scale_log2;
          if (!tile_clean && (tok >= ntok || ((bad >> (tok / p.chunk)) & 1u))) v = neg_inf;
          s[j][e] = v;
        }
      }
      // warp-local tile row maxima (rows g, g + 8)
      float mx[2];
      mx[0] = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
      mx[1] = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      }

      bool skip = false;
      bool skip_r[2] = {false, false};   // per_head: this lane's rows g, g + 8 drop the tile
      if constexpr (SKIP) {
        // tile row maxima over all four warps, then the unit-wide decision
        if (tq == 0) {
          red[(red_par * kDecConsumerWarps + warp) * 16 + g] = mx[0];
          red[(red_par * kDecConsumerWarps + warp) * 16 + g + 8] = mx[1];
        }
        named_bar_sync(1, kDecConsumerWarps * 32);
        float r[2] = {neg_inf, neg_inf};
#pragma unroll
        for (int w = 0; w < kDecConsumerWarps; ++w) {
          r[0] = fmaxf(r[0], red[(red_par * kDecConsumerWarps + w) * 16 + g]);
          r[1] = fmaxf(r[1], red[(red_par * kDecConsumerWarps + w) * 16 + g + 8]);
        }
        red_par ^= 1;
        bool row_ok = true;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const bool valid_row = rr == 0 ? row0_valid : row1_valid;
          const bool ok_r = !valid_row || r[rr] == neg_inf ||
                            (m_true[rr] != neg_inf && (r[rr] - m_true[rr]) < p.log2_lambda);
          row_ok = row_ok && ok_r;
          skip_r[rr] = ok_r;
        }
        skip = __all_sync(0xffffffffu, row_ok) != 0;
        if (p.per_head) {
          // Each query head is its own unit. A row that drops the tile gets zero
          // probabilities; its tile maximum lies below its running maximum by
          // -log2(lambda) > 0, so it cannot raise the reference either. The V
          // rows are still loaded: the group's other heads may keep them.
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
            if (!skip_r[rr]) m_true[rr] = fmaxf(m_true[rr], r[rr]);
          if (p.skip_mask && warp == 0 && tq == 0) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int row = g + 8 * rr;
              if (row < G)
                p.skip_mask[(size_t(seq) * p.Hq + kvh * G + row) * p.max_tiles + t0 / kDecTile] = skip_r[rr] ? 1 : 0;
            }
          }
          if (p.skipped_tiles && warp == 0) {
            const int n = __popc(__ballot_sync(0xffffffffu, tq == 0 && row0_valid && skip_r[0])) +
                          __popc(__ballot_sync(0xffffffffu, tq == 0 && row1_valid && skip_r[1]));
            if (lane == 0 && n) atomicAdd(p.skipped_tiles, (unsigned long long)n);
          }
        } else {
          skip_r[0] = skip_r[1] = false;
          if (!skip) {
            m_true[0] = fmaxf(m_true[0], r[0]);
            m_true[1] = fmaxf(m_true[1], r[1]);
          }
          if (p.skip_mask && warp == 0 && lane == 0)
            p.skip_mask[(size_t(seq) * p.Hkv + kvh) * p.max_tiles + t0 / kDecTile] = skip ? 1 : 0;
          if (p.skipped_tiles && warp == 0 && lane == 0 && skip) atomicAdd(p.skipped_tiles, 1ull);
        }
      }

      if (!skip) {
        // zero the V rows of masked tokens so that 0 * (stale or NaN) cannot reach O
        if (!tile_clean) {
          bool any_masked = false;
          for (int t = 0; t < 16; ++t) {
            const int tok = tok_base + t;
            const bool masked = tok >= ntok || ((bad >> (tok / p.chunk)) & 1u);
            any_masked |= masked;
            if (masked) {
              for (int c = lane; c < D / 8; c += 32)
                *reinterpret_cast<uint4*>(smem + slot * L::kStageBytes + L::kTileBytes + swz_off<D>(tok, c)) =
                    make_uint4(0, 0, 0, 0);
            }
          }
          if (any_masked) __syncwarp();
        }
        // reference maximum: raised only when the tile exceeds it by more than 2^8
        float alpha[2] = {1.f, 1.f};
        bool raised = false;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (mx[r] != neg_inf && (m_ref[r] == neg_inf || mx[r] > m_ref[r] + kDecRescaleThreshold)) {
            alpha[r] = (m_ref[r] == neg_inf) ? 0.f : fast_exp2(m_ref[r] - mx[r]);
            m_ref[r] = mx[r];
            raised = true;
          }
        }
        if (__any_sync(0xffffffffu, raised)) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
            o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
          }
          l_part[0] *= alpha[0];
          l_part[1] *= alpha[1];
          lr_part[0] *= alpha[0];
          lr_part[1] *= alpha[1];
        }
        // probabilities, packed as the A operand of P V
        uint32_t pa[4];
        {
          const float off0 = m_ref[0] == neg_inf ? 0.f : m_ref[0];
          const float off1 = m_ref[1] == neg_inf ? 0.f : m_ref[1];
          float pr[2][4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            pr[j][0] = (row0_valid && !skip_r[0]) ? fast_exp2(s[j][0] - off0) : 0.f;
            pr[j][1] = (row0_valid && !skip_r[0]) ? fast_exp2(s[j][1] - off0) : 0.f;
            pr[j][2] = (row1_valid && !skip_r[1]) ? fast_exp2(s[j][2] - off1) : 0.f;
            pr[j][3] = (row1_valid && !skip_r[1]) ? fast_exp2(s[j][3] - off1) : 0.f;
          }
          pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
          pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
          pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
          pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
          l_part[0] += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
          l_part[1] += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
          // the weights applied to V are normalised by the sum of the rounded P, so
          // they add up to one (a dominant key's P, up to 2^8 under the lagging
          // reference, would otherwise carry its bf16 rounding into the whole row)
          lr_part[0] += (bf16_lo(pa[0]) + bf16_hi(pa[0])) + (bf16_lo(pa[2]) + bf16_hi(pa[2]));
          lr_part[1] += (bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3]));
        }
        // ---- O += P V over this warp's 16 tokens
        {
          const int mi = lane >> 3, r = lane & 7;
          const int tok = tok_base + (mi & 1) * 8 + r;
#pragma unroll
          for (int n2 = 0; n2 < NT / 2; ++n2) {
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(vaddr + swz_off<D>(tok, n2 * 2 + (mi >> 1)), v0, v1, v2, v3);
            mma_bf16_16816(o[2 * n2], pa, v0, v1);
            mma_bf16_16816(o[2 * n2 + 1], pa, v2, v3);
          }
        }
        if (!tile_clean) fence_proxy_async_smem();  // zeroed rows before the next TMA write
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

      if (++slot == NS) { slot = 0; phase ^= 1u; }
      if (!last_tile) continue;

      // ---- merge the four warps' (m, l, O) in a fixed order and write the split result
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 1);
        l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 2);
        lr_part[r] += __shfl_xor_sync(0xffffffffu, lr_part[r], 1);
        lr_part[r] += __shfl_xor_sync(0xffffffffu, lr_part[r], 2);
      }
      const float inv_r0 = lr_part[0] > 0.f ? 1.f / lr_part[0] : 0.f;
      const float inv_r1 = lr_part[1] > 0.f ? 1.f / lr_part[1] : 0.f;
      if (row0_valid) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float* dst = comb_o + (warp * G + g) * D + n * 8 + 2 * tq;
          dst[0] = o[n][0] * inv_r0;
          dst[1] = o[n][1] * inv_r0;
        }
        if (tq == 0) { comb_m[warp * G + g] = m_ref[0]; comb_l[warp * G + g] = l_part[0]; }
      }
      if (row1_valid) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float* dst = comb_o + (warp * G + g + 8) * D + n * 8 + 2 * tq;
          dst[0] = o[n][2] * inv_r1;
          dst[1] = o[n][3] * inv_r1;
        }
        if (tq == 0) { comb_m[warp * G + g + 8] = m_ref[1]; comb_l[warp * G + g + 8] = l_part[1]; }
      }
      named_bar_sync(1, kDecConsumerWarps * 32);
      const int tid = threadIdx.x;
      for (int i = tid; i < G * D; i += kDecConsumerWarps * 32) {
        const int h = i / D, d = i % D;
        float M = neg_inf;
#pragma unroll
        for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, comb_m[w * G + h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kDecConsumerWarps; ++w) {
          const float mw = comb_m[w * G + h];
          const float e = (mw == neg_inf) ? 0.f : fast_exp2(mw - M);
          const float wl = e * comb_l[w * G + h];
          lsum += wl;
          osum += wl * comb_o[(w * G + h) * D + d];   // comb_o holds each warp's normalised partial
        }
        const float val = lsum > 0.f ? osum / lsum : 0.f;  // 0 only if every page was invalid
        const int hq = kvh * G + h;
        if (n_splits == 1)
          p.o[(size_t(seq) * p.Hq + hq) * D + d] = __float2bfloat16_rn(val);
        else
          p.ws_o[((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + d] = val;
        if (d == 0) {
          const float lse2 = lsum > 0.f ? M + __log2f(lsum) : neg_inf;
          if (n_splits == 1) {
            if (p.lse) p.lse[size_t(seq) * p.Hq + hq] = lse2 * 0.69314718055994531f;
          } else {
            p.ws_lse[(size_t(seq) * p.max_splits + split) * p.Hq + hq] = lse2;
          }
        }
      }
      // the next item's partials overwrite comb_* only after its first tile's
      // per-warp work; order those writes after every thread's reads above
      named_bar_sync(1, kDecConsumerWarps * 32);
    }
  }
  __syncwarp();
  __syncthreads();
}

// Combine the split partials of one (sequence, query head) per CTA -- or of
// one of DS slices of its head dimension: each partial is a normalised O row
// (fp32) with its log2-sum-exp; the result is
// sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M), M the largest lse_s. Warp w
// takes splits w, w + W, ... in chunks of kMergeChunk, loading each chunk's
// lse values and O rows together (one memory round trip per chunk), and keeps a
// running maximum; the W warps then combine in a fixed order (deterministic).
// W = 4 serves batches of many sequences; W = 16 with one slice per 32 head
// dimensions puts many partials in flight on many SMs for the few rows of a
// long single sequence. SPARSE (the tile-skip decode's chunk partials, most of
// them empty when most tiles are skipped) reads a partial's O row only when
// its log-sum-exp is finite.
constexpr int kMergeChunk = 8;   // splits per warp in flight
template <int D, int W = 4, int DS = 1, bool SPARSE = false>
__global__ void __launch_bounds__(W * 32) decode_merge_kernel(const DecodeParams p) {
  static_assert((D / 32) % DS == 0, "a slice gives each lane whole floats");
  constexpr int kMergeWarps = W;
  constexpr int DW = D / DS;    // head dimensions of this CTA's slice
  constexpr int DL = DW / 32;   // floats per lane: 4, 2 or 1
  __shared__ float sh_m[kMergeWarps], sh_w[kMergeWarps];
  __shared__ __align__(16) float sh_acc[kMergeWarps][DW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned row = blockIdx.x / unsigned(DS);
  const int slice = int(blockIdx.x % unsigned(DS));
  const int seq = int(row / unsigned(p.Hq)), hq = int(row % unsigned(p.Hq));
  const int capacity = p.max_pages * p.page_size;
  // the lengths are inputs, not results of the split kernel: read before waiting for it
  int len = __ldg(&p.seq_lens[seq]);
  len = len < 0 ? 0 : min(len, capacity);
  const int n_splits = (len + p.split_tokens - 1) / p.split_tokens;
  // every CTA waits for the split kernel (launched as its programmatic dependent), so that this
  // grid never completes before that one
  grid_dependency_wait();
  __nv_bfloat16* orow = p.o + (size_t(seq) * p.Hq + hq) * D + slice * DW;
  const float neg_inf = -__int_as_float(0x7f800000);
  if (n_splits == 1) return;  // written by the split kernel
  if (n_splits == 0) {        // a row the split kernel never writes
    for (int d = threadIdx.x; d < DW; d += blockDim.x) orow[d] = __float2bfloat16_rn(0.f);
    if (p.lse && slice == 0 && threadIdx.x == 0) p.lse[size_t(seq) * p.Hq + hq] = neg_inf;
    return;
  }
  const float* lse_base = p.ws_lse + size_t(seq) * p.max_splits * p.Hq + hq;
  const float* o_base = p.ws_o + (size_t(seq) * p.max_splits * p.Hq + hq) * D + slice * DW + lane * DL;
  const size_t o_stride = size_t(p.Hq) * D;   // floats between consecutive splits
  float acc[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) acc[d] = 0.f;
  float m = neg_inf, wsum = 0.f;
  for (int base = warp; base < n_splits; base += kMergeWarps * kMergeChunk) {
    float ls[kMergeChunk], ov[kMergeChunk][DL];
    if constexpr (SPARSE) {   // most partials empty (skipped chunks): their O rows are not read
#pragma unroll
      for (int u = 0; u < kMergeChunk; ++u) {
        const int su = base + u * kMergeWarps;
        ls[u] = su < n_splits ? lse_base[size_t(su) * p.Hq] : neg_inf;
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeChunk; ++u) {
      const int su = base + u * kMergeWarps;
      if constexpr (!SPARSE) ls[u] = neg_inf;
#pragma unroll
      for (int d = 0; d < DL; ++d) ov[u][d] = 0.f;
      if (SPARSE ? ls[u] != neg_inf : su < n_splits) {
        if constexpr (!SPARSE) ls[u] = lse_base[size_t(su) * p.Hq];
        const float* src = o_base + size_t(su) * o_stride;
        if constexpr (DL == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          ov[u][0] = t.x; ov[u][1] = t.y; ov[u][2] = t.z; ov[u][3] = t.w;
        } else if constexpr (DL == 2) {
          const float2 t = *reinterpret_cast<const float2*>(src);
          ov[u][0] = t.x; ov[u][1] = t.y;
        } else {
          ov[u][0] = *src;
        }
      }
    }
    float cm = ls[0];
#pragma unroll
    for (int u = 1; u < kMergeChunk; ++u) cm = fmaxf(cm, ls[u]);
    if (cm > m) {   // raise the running maximum (the first finite chunk rescales zeros)
      const float sc = (m == neg_inf) ? 0.f : fast_exp2(m - cm);
#pragma unroll
      for (int d = 0; d < DL; ++d) acc[d] *= sc;
      wsum *= sc;
      m = cm;
    }
#pragma unroll
    for (int u = 0; u < kMergeChunk; ++u) {
      const float w = (ls[u] == neg_inf) ? 0.f : fast_exp2(ls[u] - m);
      wsum += w;
#pragma unroll
      for (int d = 0; d < DL; ++d) acc[d] = fmaf(w, ov[u][d], acc[d]);
    }
  }
#pragma unroll
  for (int d = 0; d < DL; ++d) sh_acc[warp][lane * DL + d] = acc[d];
  if (lane == 0) { sh_m[warp] = m; sh_w[warp] = wsum; }
  __syncthreads();
  float mx = sh_m[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) mx = fmaxf(mx, sh_m[w]);
  float f[kMergeWarps];
  float wt = 0.f;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) {
    f[w] = (sh_m[w] == neg_inf) ? 0.f : fast_exp2(sh_m[w] - mx);
    wt += f[w] * sh_w[w];
  }
  const float inv = wt > 0.f ? 1.f / wt : 0.f;
  for (int d = threadIdx.x; d < DW; d += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) v = fmaf(f[w], sh_acc[w][d], v);
    orow[d] = __float2bfloat16_rn(v * inv);
  }
  if (p.lse && slice == 0 && threadIdx.x == 0)
    p.lse[size_t(seq) * p.Hq + hq] = wt > 0.f ? (mx + __log2f(wt)) * 0.69314718055994531f : neg_inf;
}

}  // namespace attn
