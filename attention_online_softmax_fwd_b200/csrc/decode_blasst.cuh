// Paged decode with the BLASST tile skip, in two passes over the head-group
// layout of decode_heads.cuh ("高效部署稀疏注意力加速方案：BLASST方法详解与实践指南",
// 架构与组件: a tile whose scores all lie far enough below the running maximum
// costs no exponentials, no Value load and no P V product).
//
// The decision for a 64-token tile needs the tile's row maxima and the running
// maximum of the tiles before it in the same split. A skipped tile lies below
// that running maximum for every row, so it never raises it: the running
// maximum at tile t is the plain prefix maximum of the tile maxima. That makes
// the decisions computable from the tile maxima alone, in any order:
//
//   pass 1 (decode_scores_kernel): work item = (chunk, sequence, group of HG KV
//     heads). K only: S^T = K q^T per 16-token stage (the transposed products of
//     the head-group kernel), written to the workspace as fp32 scaled scores in
//     log2 units, with the row maxima of every 64-token tile and of every chunk.
//   pass 2 (decode_pv_kernel): the same items. The producer warp derives the
//     decisions of the chunk's tiles from the maxima (running maximum = maximum
//     of the split's earlier chunks, then of the chunk's earlier tiles), writes
//     the decision mask and the skipped count, and streams only the kept
//     (head, tile) pairs: the tile's scores and the head's V rows. The consumers
//     take the exponentials against the largest kept score of the chunk (known
//     in advance, so no rescaling) and run P V; a chunk's partial goes to the
//     log-sum-exp merge kernel.
//
// The work decomposition (chunks) is independent of the decision units
// (splits): a single long sequence still spreads over every SM whatever
// split_tokens is. K is read once (pass 1) and V only for kept tiles (pass 2);
// the scores, 4 bytes per token and query head, are kept in L2 between passes.
#pragma once

#include "decode_heads.cuh"

namespace attn {

constexpr int kBlChunkMax = 256;                       // largest work item, tokens
constexpr int kBlChunkTiles = kBlChunkMax / kDecTile;  // 64-token tiles per work item, at most

// ---------------------------------------------------------------- pass 1

template <int D, int G, int HG>
struct BlScoresSmem {
  static constexpr int kHeadBytes = kDhChunk * D * 2;   // one head's 16 key rows
  static constexpr int kKBytes = HG * kHeadBytes;
  static constexpr int kQBytes = HG * G * D * 2;
  static constexpr int kStageBytes = kKBytes;            // a multiple of 1024
  static constexpr int kBlocks = 3;                      // resident CTAs per SM
  // the query rows of an item sit in one of two buffers of their own (items alternate)
  static constexpr int kFit = (233472 / kBlocks - 2 * kQBytes - 1024 - 2048) / (kStageBytes + 48);
  static constexpr int kStages = kFit < 6 ? kFit : 6;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kQ = kRing;
  static constexpr int kFull = kQ + 2 * kQBytes;
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kQEmpty = kEmpty + 8 * kStages;   // a query buffer was read (count HG)
  static constexpr int kInfo = kQEmpty + 16;
  static constexpr int kTotal = kInfo + 32 * kStages;
  static constexpr int kDynamic = kTotal + 1024;
  static_assert(kStages >= 2, "ring depth");
};

template <int D, int G, int HG>
__global__ void __launch_bounds__((HG + 1) * 32, 3)
    decode_scores_kernel(const __grid_constant__ CUtensorMap tm_k, const DecodeParams p, int* ticket_counter) {
  static_assert(G >= 1 && G <= 8, "transposed products: at most 8 query heads per KV head");
  using L = BlScoresSmem<D, G, HG>;
  launch_dependents();   // pass 2 may be scheduled early; it waits for this grid before reading its results
  constexpr int NS = L::kStages;
  constexpr int KS = D / 16;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  uint64_t* qempty = reinterpret_cast<uint64_t*>(smem + L::kQEmpty);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + L::kInfo);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;
  const int n_groups = p.Hkv / HG;
  const int C = p.chunk_tokens;
  const long long num_items = (long long)p.max_chunks * p.num_seqs * n_groups;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], HG);
    }
    mbar_init(&qempty[0], HG);
    mbar_init(&qempty[1], HG);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == HG) {
    // ------------------------------------------------------------ producer: K stages (and q with the first)
    if (lane == 0) tma_prefetch_desc(&tm_k);
    int slot = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pending_phase = 0;
    int qpar = 0;
    uint32_t q_phase = 0;   // bit b: phase of query buffer b
    bool ok = true;
    long long nx_item = 0;
    int nx_len = 0, nx_win = -1;
    auto fetch_next = [&]() {
      long long t = 0;
      if (lane == 0) t = atomicAdd(ticket_counter, 1);
      t = __shfl_sync(0xffffffffu, t, 0);
      nx_item = t;
      if (t < num_items) {
        int sq, ch, gr;
        dh_item_coords(t, p.num_seqs, n_groups, sq, ch, gr);
        nx_len = __ldg(&p.seq_lens[sq]);
        const int e = (((ch * C) / p.page_size) & ~31) + lane;
        nx_win = e < p.max_pages ? __ldg(&p.block_table[size_t(sq) * p.max_pages + e]) : -1;
      }
    };
    fetch_next();
    while (ok) {
      const long long item = nx_item;
      if (item >= num_items) break;
      int len = nx_len;
      int win_cur = nx_win;
      fetch_next();
      int seq, chunk, grp;
      dh_item_coords(item, p.num_seqs, n_groups, seq, chunk, grp);
      if (len > capacity || len < 0) {
        if (lane == 0 && chunk == 0 && grp == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
        len = len < 0 ? 0 : capacity;
      }
      const int t_begin = chunk * C;
      if (t_begin >= len) continue;
      const int t_end = min(t_begin + C, len);
      const int32_t* bt_row = p.block_table + size_t(seq) * p.max_pages;
      int win = (t_begin / p.page_size) >> 5;
      int win_next;
      {
        const int e = (win + 1) * 32 + lane;
        win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
      }
      const __nv_bfloat16* qsrc = p.q + (size_t(seq) * p.Hq + size_t(grp) * HG * G) * D;
      // the query buffer of this item must have been read by every consumer for the item before last
      const int qb = qpar;
      qpar ^= 1;
      if (!mbar_wait(&qempty[qb], ((q_phase >> qb) & 1u) ^ 1u, &abort_flag, p.status)) { ok = false; break; }
      q_phase ^= 1u << qb;
      uint8_t* qbuf = smem + L::kQ + qb * L::kQBytes;
      for (int t0 = t_begin; t0 < t_end && ok; t0 += kDhChunk) {
        const int e0 = t0 / p.page_size;
        if ((e0 >> 5) != win) {   // a chunk of at most 256 tokens spans at most two windows of 32 pages
          win = e0 >> 5;
          win_cur = win_next;
          const int e = (win + 1) * 32 + lane;
          win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
        }
        if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        const int page = __shfl_sync(0xffffffffu, win_cur, e0 & 31);
        if (lane == 0) {
          const bool first = t0 == t_begin;
          TileInfo ti;
          ti.seq = seq; ti.split = chunk; ti.kvh = grp; ti.t0 = t0;
          ti.ntok = min(kDhChunk, len - t0);
          ti.bad = 0;
          uint32_t bytes = first ? uint32_t(L::kQBytes) : 0u;
          if (page >= 0 && page < p.num_pages) {
            bytes += uint32_t(L::kKBytes);
          } else {
            raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
            ti.bad = 1;
          }
          ti.flags = (first ? 1 : 0) | (t0 + kDhChunk >= t_end ? 2 : 0);
          ti.len = len;
          info[slot] = ti;
          uint8_t* stage = smem + slot * L::kStageBytes;
          mbar_arrive_expect_tx(&full[slot], bytes);
          if (first) bulk_load(qbuf, qsrc, uint32_t(L::kQBytes), &full[slot]);
          if (!ti.bad) tma_load_5d(stage, &tm_k, &full[slot], 0, t0 % p.page_size, 0, grp * HG, page);
        }
        __syncwarp();
        pending |= 1u << slot;
        pending_phase = (pending_phase & ~(1u << slot)) | (phase << slot);
        if (++slot == NS) { slot = 0; phase ^= 1u; }
      }
    }
    if (ok && mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) {
      if (lane == 0) {   // end-of-work marker
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
    // ------------------------------------------------------------ consumer warp = KV head `warp` of the group
    // Lane (g, t): S^T rows (tokens) g and g + 8 of the stage, columns (query heads) 2t and 2t + 1.
    const float neg_inf = -__int_as_float(0x7f800000);
    const int g = lane >> 2, tq = lane & 3;
    const bool head_valid[2] = {2 * tq < G, 2 * tq + 1 < G};
    int slot = 0;
    uint32_t phase = 0;
    int no_abort = 0;
    bool ok = true;
    int seq = 0, chunk = 0, grp = 0;
    int qpar = 0;
    uint32_t qb[KS][2];
    const uint32_t ring_addr = smem_u32(smem);
    float tmax[2] = {neg_inf, neg_inf};   // running row maxima of the current 64-token tile
    float cmax[2] = {neg_inf, neg_inf};   // of the current chunk
    const uint64_t keep = l2_keep_policy();   // pass 2 reads the scores back from L2

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) { ok = false; break; }
      const TileInfo ti = info[slot];
      if (ti.flags & 4) break;
      if (ti.flags & 1) {
        seq = ti.seq; chunk = ti.split; grp = ti.kvh;
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(smem + L::kQ + qpar * L::kQBytes) + warp * G * (D / 2);
        const bool qv = g < G;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qb[ks][0] = qv ? qs[g * (D / 2) + ks * 8 + tq] : 0u;
          qb[ks][1] = qv ? qs[g * (D / 2) + ks * 8 + 4 + tq] : 0u;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qpar]);   // the query buffer may take the item after next
        qpar ^= 1;
        tmax[0] = tmax[1] = neg_inf;
        cmax[0] = cmax[1] = neg_inf;
      }
      float st[4] = {neg_inf, neg_inf, neg_inf, neg_inf};   // token g + 8 (e >> 1), head 2tq + (e & 1)
      if (!ti.bad) {
        float sp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint32_t kaddr = ring_addr + slot * L::kStageBytes + warp * L::kHeadBytes;
        const int mi = lane >> 3, r = lane & 7;
        const int tok = (mi & 1) * 8 + r;
        uint32_t af[KS][4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
          ldsm_x4(kaddr + dh_swz<D>(tok, ks * 2 + (mi >> 1)), af[ks][0], af[ks][1], af[ks][2], af[ks][3]);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) mma_bf16_16816(sp[ks & 1], af[ks], qb[ks][0], qb[ks][1]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tk = g + 8 * (e >> 1);
          const float v = (sp[0][e] + sp[1][e]) * p.scale_log2;
          st[e] = (!head_valid[e & 1] || tk >= ti.ntok) ? neg_inf : v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);   // the key rows are no longer needed
      if (++slot == NS) { slot = 0; phase ^= 1u; }

      // scores of this warp's query heads: [group row][token][HG][G], 16 tokens from t0
      float* srow = p.ws_s + ((size_t(seq) * (p.Hkv / HG) + grp) * p.tok64 + ti.t0) * (HG * G) + warp * G + 2 * tq;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float* dst = srow + (g + 8 * r) * (HG * G);
        if constexpr (G == 1) {
          if (tq == 0) st_keep(dst, st[2 * r], keep);
        } else {
          if (head_valid[0]) st_keep(dst, st[2 * r], st[2 * r + 1], keep);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) tmax[c] = fmaxf(tmax[c], fmaxf(st[c], st[c + 2]));
      const bool last = (ti.flags & 2) != 0;
      if (last || (ti.t0 % kDecTile) == kDecTile - kDhChunk) {
        // the 64-token tile ends here: its row maxima over the 16 token rows
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmax[c] = fmaxf(tmax[c], __shfl_xor_sync(0xffffffffu, tmax[c], 4));
          tmax[c] = fmaxf(tmax[c], __shfl_xor_sync(0xffffffffu, tmax[c], 8));
          tmax[c] = fmaxf(tmax[c], __shfl_xor_sync(0xffffffffu, tmax[c], 16));
          cmax[c] = fmaxf(cmax[c], tmax[c]);
          if (g == 0 && head_valid[c]) {
            const int hq = (grp * HG + warp) * G + 2 * tq + c;
            p.ws_tmax[(size_t(seq) * p.Hq + hq) * p.max_tiles + ti.t0 / kDecTile] = tmax[c];
            if (last) p.ws_cmax[(size_t(seq) * p.Hq + hq) * p.max_chunks + chunk] = cmax[c];
          }
          tmax[c] = neg_inf;
        }
      }
    }
  }
  __syncwarp();
  __syncthreads();
}

// ---------------------------------------------------------------- between the passes (long splits)

// The exclusive running maximum of the chunk maxima within each decision split:
// ws_cpre[row][ch] = maximum of ws_cmax[row][j] over the chunks j < ch of ch's split,
// -inf for a split's first chunk. One warp per (sequence, query head) row: a segmented
// max-scan over 32 chunks at a time (segments = splits), carried from block to block,
// with kScanBatch blocks loaded before they are scanned.
constexpr int kScanWarps = 4;
constexpr int kScanBatch = 8;
__global__ void __launch_bounds__(kScanWarps * 32) decode_chunk_prefix_kernel(const DecodeParams p) {
  launch_dependents();     // pass 2 may be scheduled early; it waits for this grid
  grid_dependency_wait();  // pass 1's chunk maxima
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kScanWarps + warp;   // seq * Hq + hq
  if (row >= (long long)p.num_seqs * p.Hq) return;
  const float neg_inf = -__int_as_float(0x7f800000);
  const int seq = int(row / p.Hq);
  const int capacity = p.max_pages * p.page_size;
  int len = __ldg(&p.seq_lens[seq]);
  len = len < 0 ? 0 : min(len, capacity);
  const int C = p.chunk_tokens;
  const int nch = (len + C - 1) / C;
  const int cps = p.split_tokens / C;   // chunks per split
  const float* cm = p.ws_cmax + size_t(row) * p.max_chunks;
  float* cp = p.ws_cpre + size_t(row) * p.max_chunks;
  float carry = neg_inf;
  for (int base = 0; base < nch; base += 32 * kScanBatch) {
    float v[kScanBatch];
#pragma unroll
    for (int b = 0; b < kScanBatch; ++b) {
      const int ch = base + b * 32 + lane;
      v[b] = ch < nch ? cm[ch] : neg_inf;
    }
#pragma unroll
    for (int b = 0; b < kScanBatch; ++b) {
      if (base + b * 32 >= nch) break;
      const int ch = base + b * 32 + lane;
      const bool start = ch % cps == 0;
      // inclusive scan: (value, "a split starts in my window") combined with the window to the left
      float inc = v[b];
      int fl = start ? 1 : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const float ov = __shfl_up_sync(0xffffffffu, inc, d);
        const int of = __shfl_up_sync(0xffffffffu, fl, d);
        if (lane >= d) {
          if (!fl) inc = fmaxf(inc, ov);
          fl |= of;
        }
      }
      if (!fl) inc = fmaxf(inc, carry);   // no split start between the block's start and this chunk
      const float left = __shfl_up_sync(0xffffffffu, inc, 1);
      if (ch < nch) cp[ch] = start ? neg_inf : (lane == 0 ? carry : left);
      carry = __shfl_sync(0xffffffffu, inc, 31);
    }
  }
}

// ---------------------------------------------------------------- pass 2

// What the pass-2 producer tells the consumers about a stage.
struct BlStageInfo {
  int seq, chunk, grp, t0;
  int ntok;        // valid tokens of the stage from t0
  int flags;       // 1 first stage of the item, 2 last, 4 end of work, 8 nothing to read in this stage
  int len;         // sequence length (clamped)
  int load;        // bit w: the stage holds KV head w's scores and V rows
  uint32_t keep;   // bit r: group row r (KV head r / G, query head r % G) keeps the stage's tile
  float mref[32];  // first stage: per group row, the largest score of the chunk's kept tiles
};

template <int D, int G, int HG>
struct BlPvSmem {
  static constexpr int kHeadBytes = kDhChunk * D * 2;     // one head's 16 V rows
  static constexpr int kVBytes = HG * kHeadBytes;
  static constexpr int kSBytes = kDhChunk * HG * G * 4;   // the stage's scores [16][HG][G]
  static constexpr int kStageBytes = (kVBytes + kSBytes + 1023) / 1024 * 1024;
  static constexpr int kInfoBytes = (int(sizeof(BlStageInfo)) + 15) / 16 * 16;
  static constexpr int kBlocks = 3;
  static constexpr int kFit = (233472 / kBlocks - 1024 - 2048) / (kStageBytes + 16 + kInfoBytes);
  static constexpr int kStages = kFit < 6 ? kFit : 6;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kFull = kRing;
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kInfo = kEmpty + 8 * kStages;
  static constexpr int kTotal = kInfo + kInfoBytes * kStages;
  static constexpr int kDynamic = kTotal + 1024;
  static_assert(kStages >= 2, "ring depth");
  static_assert(HG * G <= 32, "one producer lane per group row");
};

template <int D, int G, int HG, bool PER_HEAD>
__global__ void __launch_bounds__((HG + 1) * 32, 3)
    decode_pv_kernel(const __grid_constant__ CUtensorMap tm_v_group, const __grid_constant__ CUtensorMap tm_v_head,
                     const DecodeParams p, int* ticket_counter) {
  static_assert(G >= 1 && G <= 8, "transposed products: at most 8 query heads per KV head");
  using L = BlPvSmem<D, G, HG>;
  launch_dependents();      // the merge kernel may be scheduled early; it waits for this grid
  grid_dependency_wait();   // pass 1's scores and maxima are complete and visible (every role waits, so
                            // that no pipeline wait below starts its clock before pass 1 has finished)
  constexpr int NS = L::kStages;
  constexpr int R = HG * G;                       // query heads (rows) of a group
  constexpr uint32_t kUnit = (1u << G) - 1u;      // the rows of one KV head, at bit 0

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  BlStageInfo* info = reinterpret_cast<BlStageInfo*>(smem + L::kInfo);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;
  const int n_groups = p.Hkv / HG;
  const int C = p.chunk_tokens;     // pass-1 chunk (the granularity of the chunk maxima)
  const int C2 = p.chunk2_tokens;   // this pass's work item, a whole number of pass-1 chunks
  const long long num_items = (long long)p.max_chunks2 * p.num_seqs * n_groups;
  const float neg_inf = -__int_as_float(0x7f800000);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], HG);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == HG) {
    // ------------------------------------------------------------ producer: decisions, then kept S and V
    if (lane == 0) {
      tma_prefetch_desc(&tm_v_group);
      tma_prefetch_desc(&tm_v_head);
    }
    const bool active = p.log2_lambda != neg_inf;   // lambda > 0
    int slot = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pending_phase = 0;
    bool ok = true;
    // The next item (ticket), its length and first block-table window, and the maxima its
    // decisions need -- its tiles' row maxima and the first sixteen chunk maxima of its split
    // before it -- are all loaded one item ahead, so that an item starts without a round trip.
    // Lane r < R stands for group row r (query head grp * R + r).
    long long nx_item = 0;
    int nx_len = 0, nx_win = -1;
    float nx_tm[kBlChunkTiles];
    float nx_cm[16];
    auto fetch_next = [&]() {
      long long t = 0;
      if (lane == 0) t = atomicAdd(ticket_counter, 1);
      t = __shfl_sync(0xffffffffu, t, 0);
      nx_item = t;
      if (t < num_items) {
        int sq, ch, gr;
        dh_item_coords(t, p.num_seqs, n_groups, sq, ch, gr);
        nx_len = __ldg(&p.seq_lens[sq]);
        const int e = (((ch * C2) / p.page_size) & ~31) + lane;
        nx_win = e < p.max_pages ? __ldg(&p.block_table[size_t(sq) * p.max_pages + e]) : -1;
        const size_t rb = size_t(sq) * p.Hq + (lane < R ? gr * R + lane : 0);
        const int ta = ch * C2 / kDecTile;
        const int c1 = ch * C2 / C;   // the item's first pass-1 chunk
#pragma unroll
        for (int i = 0; i < kBlChunkTiles; ++i)   // tiles past the sequence end are read, never used
          nx_tm[i] = (lane < R && ta + i < p.max_tiles) ? p.ws_tmax[rb * p.max_tiles + ta + i] : neg_inf;
        if (p.ws_cpre) {   // long splits: the running maximum at the chunk start, computed between the passes
          nx_cm[0] = lane < R ? p.ws_cpre[rb * p.max_chunks + c1] : neg_inf;
#pragma unroll
          for (int u = 1; u < 16; ++u) nx_cm[u] = neg_inf;
        } else {
          const int j0 = (ch * C2 / p.split_tokens) * (p.split_tokens / C);
#pragma unroll
          for (int u = 0; u < 16; ++u)
            nx_cm[u] = (lane < R && j0 + u < c1) ? p.ws_cmax[rb * p.max_chunks + j0 + u] : neg_inf;
        }
      }
    };
    fetch_next();
    while (ok) {
      const long long item = nx_item;
      if (item >= num_items) break;
      int len = nx_len;
      int win_cur = nx_win;
      float tm[kBlChunkTiles];
      float m = neg_inf;   // running maximum at the chunk start: the split's earlier chunks' maxima
#pragma unroll
      for (int i = 0; i < kBlChunkTiles; ++i) tm[i] = nx_tm[i];
#pragma unroll
      for (int u = 0; u < 16; ++u) m = fmaxf(m, nx_cm[u]);
      fetch_next();
      int seq, chunk, grp;
      dh_item_coords(item, p.num_seqs, n_groups, seq, chunk, grp);
      if (len > capacity || len < 0) len = len < 0 ? 0 : capacity;   // reported by pass 1
      const int t_begin = chunk * C2;
      if (t_begin >= len) continue;
      const int t_end = min(t_begin + C2, len);

      // ---- decisions of the chunk's tiles
      const int hq = grp * R + lane;
      const size_t row_base = (size_t(seq) * p.Hq + (lane < R ? hq : 0));
      const int nt = (t_end - t_begin + kDecTile - 1) / kDecTile;
#pragma unroll
      for (int i = 0; i < kBlChunkTiles; ++i)
        if (i >= nt) tm[i] = neg_inf;
      if (!p.ws_cpre) {
        // chunk maxima beyond the first sixteen of the split (splits of 17 to 32 chunks; longer ones
        // have the running maximum at each chunk start computed between the passes)
        const int j0 = (t_begin / p.split_tokens) * (p.split_tokens / C) + 16;
        const float* cm = p.ws_cmax + row_base * p.max_chunks;
        const int c1 = t_begin / C;
        for (int jb = j0; jb < c1; jb += 16) {
          float v[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] = (lane < R && jb + u < c1) ? cm[jb + u] : neg_inf;
#pragma unroll
          for (int u = 0; u < 16; ++u) m = fmaxf(m, v[u]);
        }
      }
      uint32_t keep_t[kBlChunkTiles];
      float mref = neg_inf;
      int n_skipped = 0;
      int last_kept = -1;
#pragma unroll
      for (int i = 0; i < kBlChunkTiles; ++i) {
        keep_t[i] = 0;
        if (i >= nt) continue;
        const int t = t_begin / kDecTile + i;
        if ((t * kDecTile) % p.split_tokens == 0) m = neg_inf;   // a decision split starts with this tile
        const float T = tm[i];
        // the rule for one row: no visible score in the tile, or a finite running maximum that the
        // tile stays below by more than -log2(lambda)
        const bool row_ok = lane >= R || T == neg_inf || (m != neg_inf && (T - m) < p.log2_lambda);
        bool kept;
        if constexpr (PER_HEAD) {
          kept = !(active && row_ok);
        } else {
          const uint32_t okb = __ballot_sync(0xffffffffu, row_ok);
          const uint32_t um = kUnit << ((lane / G) * G);
          kept = !(active && (okb & um) == um);
        }
        kept = kept && lane < R;
        if (kept) mref = fmaxf(mref, T);
        m = fmaxf(m, T);   // a dropped tile lies below m and cannot raise it
        keep_t[i] = __ballot_sync(0xffffffffu, kept);
        if (keep_t[i]) last_kept = i;
        const bool unit_lane = lane < R && (PER_HEAD || lane % G == 0);
        if (unit_lane && p.skip_mask) {
          const size_t unit = PER_HEAD ? (size_t(seq) * p.Hq + hq) : (size_t(seq) * p.Hkv + grp * HG + lane / G);
          p.skip_mask[unit * p.max_tiles + t] = kept ? 0 : 1;
        }
        n_skipped += __popc(__ballot_sync(0xffffffffu, unit_lane && !kept));
      }
      if (p.skipped_tiles && lane == 0 && n_skipped) atomicAdd(p.skipped_tiles, (unsigned long long)n_skipped);
      if (last_kept < 0 && len > C2) {
        // nothing kept (only with lambda > 0): the chunk's partial is empty, and the merge reads no O
        // row whose log-sum-exp is -inf -- written here, with no stage for the consumers
        if (lane < R) p.ws_lse[(size_t(seq) * p.max_chunks2 + chunk) * p.Hq + hq] = neg_inf;
        continue;
      }

      // ---- stream the stages of the kept tiles (one empty stage if the chunk keeps nothing)
      const int32_t* bt_row = p.block_table + size_t(seq) * p.max_pages;
      int win = (t_begin / p.page_size) >> 5;
      int win_next;
      {
        const int e = (win + 1) * 32 + lane;
        win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
      }
      bool first = true;
      const float* s_item = p.ws_s + (size_t(seq) * n_groups + grp) * p.tok64 * R;
      for (int i = 0; i <= (last_kept < 0 ? 0 : last_kept) && ok; ++i) {
        if (last_kept >= 0 && keep_t[i] == 0) continue;
        const int s0 = t_begin + i * kDecTile;
        const int s1 = last_kept < 0 ? s0 + 1 : min(s0 + kDecTile, t_end);
        for (int t0 = s0; t0 < s1 && ok; t0 += kDhChunk) {
          const int e0 = t0 / p.page_size;
          if ((e0 >> 5) != win) {   // at most two windows per chunk; skipped tiles never jump a window
            win = e0 >> 5;
            win_cur = win_next;
            const int e = (win + 1) * 32 + lane;
            win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
          }
          if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
          const int page = __shfl_sync(0xffffffffu, win_cur, e0 & 31);
          const bool last = last_kept < 0 || (i == last_kept && t0 + kDhChunk >= s1);
          BlStageInfo& ti = info[slot];
          if (first && lane < R) ti.mref[lane] = mref;
          __syncwarp();   // every lane's reference maximum is written before lane 0 releases the stage
          if (lane == 0) {
            ti.seq = seq; ti.chunk = chunk; ti.grp = grp; ti.t0 = t0;
            ti.ntok = last_kept < 0 ? 0 : min(kDhChunk, len - t0);
            ti.len = len;
            ti.keep = keep_t[i];
            int load = 0;
#pragma unroll
            for (int w = 0; w < HG; ++w)
              if ((keep_t[i] >> (w * G)) & kUnit) load |= 1 << w;
            const bool nodata = last_kept < 0 || !(page >= 0 && page < p.num_pages);
            if (nodata) load = 0;
            ti.load = load;
            ti.flags = (first ? 1 : 0) | (last ? 2 : 0) | (nodata ? 8 : 0);
            uint32_t bytes = load ? uint32_t(L::kSBytes) + uint32_t(__popc(load)) * uint32_t(L::kHeadBytes) : 0u;
            uint8_t* stage = smem + slot * L::kStageBytes;
            mbar_arrive_expect_tx(&full[slot], bytes);
            if (load) {
              bulk_load(stage + L::kVBytes, s_item + size_t(t0) * R, uint32_t(L::kSBytes), &full[slot]);
              const int in_page = t0 % p.page_size;
              if (load == (1 << HG) - 1) {
                tma_load_5d(stage, &tm_v_group, &full[slot], 0, in_page, 0, grp * HG, page);
              } else {
#pragma unroll
                for (int w = 0; w < HG; ++w)
                  if ((load >> w) & 1)
                    tma_load_5d(stage + w * L::kHeadBytes, &tm_v_head, &full[slot], 0, in_page, 0, grp * HG + w, page);
              }
            }
          }
          __syncwarp();
          first = false;
          pending |= 1u << slot;
          pending_phase = (pending_phase & ~(1u << slot)) | (phase << slot);
          if (++slot == NS) { slot = 0; phase ^= 1u; }
        }
      }
    }
    if (ok && mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) {
      if (lane == 0) {   // end-of-work marker
        info[slot].flags = 4;
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
    // ------------------------------------------------------------ consumer warp = KV head `warp` of the group
    // O^T += V^T P^T as in the head-group kernel: lane (g, t) holds P^T for tokens 2t, 2t + 1 (+ 8) of
    // query head g and O^T rows (head dims) 16m + g, 16m + g + 8 of heads 2t, 2t + 1.
    const int g = lane >> 2, tq = lane & 3;
    const bool head_valid[2] = {2 * tq < G, 2 * tq + 1 < G};
    int slot = 0;
    uint32_t phase = 0;
    int no_abort = 0;
    bool ok = true;
    int seq = 0, chunk = 0, grp = 0, len = 0;
    constexpr int MT = D / 16;
    float o[MT][4];
    float mr[2] = {neg_inf, neg_inf};
    float l_part[2] = {0.f, 0.f};
    float lr_part[2] = {0.f, 0.f};
    const uint32_t ring_addr = smem_u32(smem);

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) { ok = false; break; }
      const BlStageInfo& ti = info[slot];
      const int flags = ti.flags;
      if (flags & 4) break;
      if (flags & 1) {
        seq = ti.seq; chunk = ti.chunk; grp = ti.grp; len = ti.len;
#pragma unroll
        for (int c = 0; c < 2; ++c) mr[c] = head_valid[c] ? ti.mref[warp * G + 2 * tq + c] : neg_inf;
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        l_part[0] = l_part[1] = 0.f;
        lr_part[0] = lr_part[1] = 0.f;
      }
      const bool last = (flags & 2) != 0;
      if (!(flags & 8) && ((ti.load >> warp) & 1)) {
        const int ntok = ti.ntok;
        const uint32_t kept = ti.keep >> (warp * G + 2 * tq);
        const float* sb = reinterpret_cast<const float*>(smem + slot * L::kStageBytes + L::kVBytes) + warp * G + 2 * tq;
        float st[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = e & 1;
          const bool use = head_valid[c] && ((kept >> c) & 1u);
          st[e] = use ? sb[(g + 8 * (e >> 1)) * R + c] : neg_inf;
        }
        const float off[2] = {mr[0] == neg_inf ? 0.f : mr[0], mr[1] == neg_inf ? 0.f : mr[1]};
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(st[e] - off[e & 1]);
        l_part[0] += pr[0] + pr[2];
        l_part[1] += pr[1] + pr[3];
        const uint32_t x0 = pack_bf16x2(pr[0], pr[1]);   // token g, heads 2tq, 2tq + 1
        const uint32_t x1 = pack_bf16x2(pr[2], pr[3]);   // token g + 8
        lr_part[0] += bf16_lo(x0) + bf16_lo(x1);
        lr_part[1] += bf16_hi(x0) + bf16_hi(x1);
        const uint32_t pb0 = movmatrix_trans(x0), pb1 = movmatrix_trans(x1);
        const uint32_t vaddr = ring_addr + slot * L::kStageBytes + warp * L::kHeadBytes;
        const int mi = lane >> 3, r = lane & 7;
        const int tok = (mi >> 1) * 8 + r;
        // rows past the end are zeroed so that 0 * (stale or NaN) cannot reach O
        const uint32_t mk0 = (2 * tq < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 1 < ntok ? 0xFFFF0000u : 0u);
        const uint32_t mk1 = (2 * tq + 8 < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 9 < ntok ? 0xFFFF0000u : 0u);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint32_t a[4];
          ldsm_x4_t(vaddr + dh_swz<D>(tok, 2 * m + (mi & 1)), a[0], a[1], a[2], a[3]);
          a[0] &= mk0; a[1] &= mk0; a[2] &= mk1; a[3] &= mk1;
          mma_bf16_16816(o[m], a, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == NS) { slot = 0; phase ^= 1u; }
      if (!last) continue;

      // ---- the chunk's result for heads 2tq, 2tq + 1 of this warp's KV head
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 4);
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 8);
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 16);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 4);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 8);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 16);
      }
      const int n_chunks = (len + C2 - 1) / C2;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (!head_valid[c]) continue;
        const int hq = (grp * HG + warp) * G + 2 * tq + c;
        const float lsum = l_part[c];
        const float inv = lr_part[c] > 0.f ? 1.f / lr_part[c] : 0.f;
        if (n_chunks == 1) {
          __nv_bfloat16* dst = p.o + (size_t(seq) * p.Hq + hq) * D + g;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            dst[16 * m] = __float2bfloat16_rn(o[m][c] * inv);
            dst[16 * m + 8] = __float2bfloat16_rn(o[m][c + 2] * inv);
          }
          if (p.lse && g == 0)
            p.lse[size_t(seq) * p.Hq + hq] = lsum > 0.f ? (mr[c] + __log2f(lsum)) * 0.69314718055994531f : neg_inf;
        } else {
          const uint64_t keep = l2_keep_policy();
          float* dst = p.ws_o + ((size_t(seq) * p.max_chunks2 + chunk) * p.Hq + hq) * D + g;
          // with lambda > 0 the merge reads an O row only when its log-sum-exp is finite
          if (lsum > 0.f || p.log2_lambda == neg_inf) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              st_keep(dst + 16 * m, o[m][c] * inv, keep);
              st_keep(dst + 16 * m + 8, o[m][c + 2] * inv, keep);
            }
          }
          if (g == 0)
            st_keep(&p.ws_lse[(size_t(seq) * p.max_chunks2 + chunk) * p.Hq + hq],
                    lsum > 0.f ? mr[c] + __log2f(lsum) : neg_inf, keep);
        }
      }
    }
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace attn
