// Paged decode with the BLASST tile skip in a single pass over the head-group
// layout of decode_heads.cuh ("高效部署稀疏注意力加速方案：BLASST方法详解与实践指南",
// 架构与组件: a skipped tile costs no exponentials, no Value load and no P V
// product).
//
// Work item = (split, sequence, group of HG KV heads), as in the dense
// head-group kernel, and consumer warp h walks the split in token order for KV
// head h: the running maximum that the skip rule compares a tile against is the
// warp's own. The producer warp streams K only, 16-token stages of all HG heads.
// A consumer warp scores the stages of a 64-token tile (S^T = K q^T, the
// transposed products), decides the tile from its row maxima and the split's
// running maximum (maximum of the earlier tiles' row maxima), and only then asks
// for the tile's V rows of its own head: one 16-token TMA copy per stage, issued
// by the warp into a tile buffer of its own (kVBufs of them). A kept tile's P V
// runs when its buffer is needed again, kVBufs kept tiles later, so that the V
// copy lands while the warp scores on; a split's last tiles are finished at the
// end of the next split's first tile, the warp keeping the split's accumulators
// until then. Split partials go to the log-sum-exp merge kernel like the dense
// kernel's. One buffer per warp at three CTAs per SM measured faster than two
// buffers at two CTAs per SM: the stream depth is set by the CTAs' K rings.
//
// The two-pass kernels (decode_blasst.cuh) decouple the work items from the
// decision splits; this one needs enough splits to fill the GPU, and in return
// reads K and the kept V exactly once with no scores in between.
#pragma once

#include "decode_heads.cuh"

namespace attn {

// What the producer tells the consumers about a K stage.
struct alignas(16) GateInfo {
  int seq, split, grp, t0;
  int ntok;   // valid tokens of the stage from t0
  int bad;    // 1: the page was outside the pool (not loaded)
  int flags;  // bit 0: first stage of the item (its query rows are in the query buffer), bit 1: last stage,
              // bit 2: no stage, this CTA's work is done
  int len;    // sequence length (clamped to the block table's capacity)
  int page;   // physical page of the stage (for the V copies)
  int pad[3];
};

template <int D, int G, int HG>
struct GateSmem {
  static constexpr int kHeadBytes = kDhChunk * D * 2;                  // one head's 16 rows of K or V
  static constexpr int kKBytes = HG * kHeadBytes;                      // a K stage
  static constexpr int kTileStages = kDecTile / kDhChunk;              // 4 stages per decision tile
  static constexpr int kVWarp = kTileStages * kHeadBytes;              // one head's V rows of a tile
  static constexpr int kQBytes = HG * G * D * 2;
  static constexpr int kVBufs = 1;                                     // tile buffers per consumer warp
  static constexpr int kBlocks = HG == 1 ? 5 : 3;                      // resident CTAs per SM
  static constexpr int kInfoBytes = int(sizeof(GateInfo));
  static constexpr int kFixed = HG * kVBufs * kVWarp + 2 * kQBytes + 16 + 8 * HG * kVBufs + 32 * HG + 16;
  static constexpr int kFit = (233472 / kBlocks - 3072 - kFixed) / (kKBytes + 16 + kInfoBytes);
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kV = 0;                                         // [HG][kVBufs][4 stages][head block]
  static constexpr int kRing = kV + HG * kVBufs * kVWarp;              // K stages
  static constexpr int kQ = kRing + kStages * kKBytes;                 // two query buffers (items alternate)
  static constexpr int kFull = kQ + 2 * kQBytes;
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kQEmpty = kEmpty + 8 * kStages;                 // a query buffer was read (count HG)
  static constexpr int kVFull = kQEmpty + 16;                          // per tile buffer: its V copies landed
  static constexpr int kWarpNote = (kVFull + 8 * HG * kVBufs + 15) / 16 * 16;   // per consumer warp: 8 ints
  static constexpr int kInfo = kWarpNote + 32 * HG;
  static constexpr int kTotal = kInfo + kInfoBytes * kStages;
  static constexpr int kDynamic = kTotal + 1024;
  static_assert(kStages >= 2, "ring depth");
  static_assert(kDynamic <= 233472 / kBlocks - 2048, "shared memory per block");
};

template <int D, int G, int HG, bool PER_HEAD>
__global__ void __launch_bounds__((HG + 1) * 32, GateSmem<D, G, HG>::kBlocks)
    decode_gate_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DecodeParams p, int* ticket_counter) {
  static_assert(G >= 1 && G <= 8, "transposed products: at most 8 query heads per KV head");
  using L = GateSmem<D, G, HG>;
  launch_dependents();   // let the merge kernel be scheduled early; it waits for this grid to finish
  constexpr int NS = L::kStages;
  constexpr int KS = D / 16;
  constexpr int MT = D / 16;   // m-tiles of O^T
  constexpr int TS = L::kTileStages;
  constexpr int NB = L::kVBufs;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  uint64_t* qempty = reinterpret_cast<uint64_t*>(smem + L::kQEmpty);
  uint64_t* vfull = reinterpret_cast<uint64_t*>(smem + L::kVFull);
  GateInfo* info = reinterpret_cast<GateInfo*>(smem + L::kInfo);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;
  const int n_groups = p.Hkv / HG;
  const long long num_items = (long long)p.max_splits * p.num_seqs * n_groups;
  const float neg_inf = -__int_as_float(0x7f800000);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], HG);
    }
    mbar_init(&qempty[0], HG);
    mbar_init(&qempty[1], HG);
    for (int w = 0; w < HG * NB; ++w) mbar_init(&vfull[w], 1);
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
    // next item (ticket), its length and first block-table window, one item ahead
    long long nx_item = 0;
    int nx_len = 0, nx_win = -1;
    auto fetch_next = [&]() {
      long long t = 0;
      if (lane == 0) t = atomicAdd(ticket_counter, 1);
      t = __shfl_sync(0xffffffffu, t, 0);
      nx_item = t;
      if (t < num_items) {
        int sq, sp, gr;
        dh_item_coords(t, p.num_seqs, n_groups, sq, sp, gr);
        nx_len = __ldg(&p.seq_lens[sq]);
        const int e = (((sp * p.split_tokens) / p.page_size) & ~31) + lane;
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
      int seq, split, grp;
      dh_item_coords(item, p.num_seqs, n_groups, seq, split, grp);
      if (len > capacity || len < 0) {
        if (lane == 0 && split == 0 && grp == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
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
      const __nv_bfloat16* qsrc = p.q + (size_t(seq) * p.Hq + size_t(grp) * HG * G) * D;
      // the query buffer of this item must have been read by every consumer for the item before last
      const int qb = qpar;
      qpar ^= 1;
      if (!mbar_wait(&qempty[qb], ((q_phase >> qb) & 1u) ^ 1u, &abort_flag, p.status)) { ok = false; break; }
      q_phase ^= 1u << qb;
      uint8_t* qbuf = smem + L::kQ + qb * L::kQBytes;
      for (int t0 = t_begin; t0 < t_end && ok; t0 += kDhChunk) {
        const int e0 = t0 / p.page_size;
        if ((e0 >> 5) != win) {   // a stage advances by at most one page, so by at most one window
          win = e0 >> 5;
          win_cur = win_next;
          const int e = (win + 1) * 32 + lane;
          win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
        }
        if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        const int page = __shfl_sync(0xffffffffu, win_cur, e0 & 31);
        if (lane == 0) {
          const bool first = t0 == t_begin;
          GateInfo ti;
          ti.seq = seq; ti.split = split; ti.grp = grp; ti.t0 = t0;
          ti.ntok = min(kDhChunk, len - t0);
          ti.bad = 0;
          ti.page = page;
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
          uint8_t* stage = smem + L::kRing + slot * L::kKBytes;
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
        GateInfo ti{};
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
    // Lane (g, t): S^T rows (tokens) g and g + 8 of a stage, columns (query heads) 2t and 2t + 1; P^T operand
    // tokens 2t, 2t + 1 (+ 8) of query head g; O^T rows (head dims) 16m + g, 16m + g + 8 of heads 2t, 2t + 1.
    const int g = lane >> 2, tq = lane & 3;
    const bool head_valid[2] = {2 * tq < G, 2 * tq + 1 < G};
    const bool active = p.log2_lambda != neg_inf;   // lambda > 0
    int slot = 0;
    uint32_t phase = 0;
    int no_abort = 0;
    bool ok = true;
    int qpar = 0;
    uint32_t qb[KS][2];
    float o[MT][4];
    float m_ref[2] = {neg_inf, neg_inf};   // lagging reference of the exponentials (heads 2tq, 2tq + 1)
    float m_run[2] = {neg_inf, neg_inf};   // the split's running maximum of tile row maxima (decisions)
    float l_part[2] = {0.f, 0.f};
    float lr_part[2] = {0.f, 0.f};
    float st[TS][4];                       // the current tile's S^T, per stage
    uint32_t t_ntok = 0;                   // and valid tokens, 5 bits per stage (0: nothing loaded)
    // Kept tiles whose V rows are on the way, oldest first, in the warp's NB tile buffers: their P^T
    // and valid tokens per stage. A tile's P V runs when its buffer is needed again (NB tiles later),
    // when the reference maximum rises, or at the first tile after its split's end.
    uint32_t pb[NB][TS][2];
    uint32_t pv_ntok[NB];
    int vq_head = 0, vq_n = 0;
    uint32_t v_phase = 0;                  // bit b: phase of buffer b's barrier
    // A finished split keeps its accumulators (o, l_part, lr_part, m_ref) while the warp scores the
    // next split's first tile: that tile's exponentials and P V come later, so the accumulators are
    // free until the split's last P V (its V rows had the tile's K stream to land) and its result.
    bool fin_pending = false;
    // this warp's notes in shared memory: [0, 4) the current tile's pages (lane 0 issues the V copies),
    // [4, 8) the finished split's sequence, group, split and split count
    int* note = reinterpret_cast<int*>(smem + L::kWarpNote) + warp * 8;
    uint32_t n_skipped = 0;   // decisions of this lane (one warp sees far fewer than 2^32)
    uint64_t* my_vfull = vfull + warp * NB;
    uint8_t* vbuf = smem + L::kV + warp * NB * L::kVWarp;
    const uint32_t ring_addr = smem_u32(smem + L::kRing);
    const uint32_t vbuf_addr = smem_u32(vbuf);
#pragma unroll
    for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
#pragma unroll
    for (int j = 0; j < TS; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[j][e] = neg_inf;
#pragma unroll
    for (int b = 0; b < NB; ++b) pv_ntok[b] = 0;

    // O^T += V^T P^T for the oldest pending tile, once its V rows have landed
    auto pv_oldest = [&]() -> bool {
      const int b = vq_head;
      if (!mbar_wait(&my_vfull[b], (v_phase >> b) & 1u, reinterpret_cast<volatile int*>(&no_abort), p.status))
        return false;
      v_phase ^= 1u << b;
      vq_head = b + 1 == NB ? 0 : b + 1;
      --vq_n;
      const int mi = lane >> 3, r = lane & 7;
      const int tok = (mi >> 1) * 8 + r;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        if (bb != b) continue;
#pragma unroll
        for (int j = 0; j < TS; ++j) {
          const int ntok = int((pv_ntok[bb] >> (5 * j)) & 31u);
          if (ntok == 0) continue;
          // rows past the end are zeroed so that 0 * (stale or NaN) cannot reach O
          const uint32_t mk0 = (2 * tq < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 1 < ntok ? 0xFFFF0000u : 0u);
          const uint32_t mk1 = (2 * tq + 8 < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 9 < ntok ? 0xFFFF0000u : 0u);
          const uint32_t base = vbuf_addr + bb * L::kVWarp + j * L::kHeadBytes;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            uint32_t a[4];
            ldsm_x4_t(base + dh_swz<D>(tok, 2 * m + (mi & 1)), a[0], a[1], a[2], a[3]);
            a[0] &= mk0; a[1] &= mk0; a[2] &= mk1; a[3] &= mk1;
            mma_bf16_16816(o[m], a, pb[bb][j][0], pb[bb][j][1]);
          }
        }
      }
      return true;
    };

    // a split's result for heads 2tq, 2tq + 1 of this warp's KV head, then the accumulators cleared
    auto write_split = [&](int sq, int gr, int spl, int nspl) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 4);
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 8);
        l_part[c] += __shfl_xor_sync(0xffffffffu, l_part[c], 16);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 4);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 8);
        lr_part[c] += __shfl_xor_sync(0xffffffffu, lr_part[c], 16);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (!head_valid[c]) continue;
        const int hq = (gr * HG + warp) * G + 2 * tq + c;
        const float lsum = l_part[c];
        const float inv = lr_part[c] > 0.f ? 1.f / lr_part[c] : 0.f;   // 0 when the split kept nothing
        if (nspl == 1) {
          __nv_bfloat16* dst = p.o + (size_t(sq) * p.Hq + hq) * D + g;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            dst[16 * m] = __float2bfloat16_rn(o[m][c] * inv);
            dst[16 * m + 8] = __float2bfloat16_rn(o[m][c + 2] * inv);
          }
          if (p.lse && g == 0)
            p.lse[size_t(sq) * p.Hq + hq] = lsum > 0.f ? (m_ref[c] + __log2f(lsum)) * 0.69314718055994531f : neg_inf;
        } else {
          const uint64_t keep_pol = l2_keep_policy();   // the merge reads these back after the KV stream
          float* dst = p.ws_o + ((size_t(sq) * p.max_splits + spl) * p.Hq + hq) * D + g;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            st_keep(dst + 16 * m, o[m][c] * inv, keep_pol);
            st_keep(dst + 16 * m + 8, o[m][c + 2] * inv, keep_pol);
          }
          if (g == 0)
            st_keep(&p.ws_lse[(size_t(sq) * p.max_splits + spl) * p.Hq + hq],
                    lsum > 0.f ? m_ref[c] + __log2f(lsum) : neg_inf, keep_pol);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
      l_part[0] = l_part[1] = 0.f;
      lr_part[0] = lr_part[1] = 0.f;
      m_ref[0] = m_ref[1] = neg_inf;
    };

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) { ok = false; break; }
      const GateInfo ti = info[slot];
      if (ti.flags & 4) break;
      if (ti.flags & 1) {
        m_run[0] = m_run[1] = neg_inf;
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
      }
      // ---- S^T = K q^T for the stage's 16 tokens
      float s4[4] = {neg_inf, neg_inf, neg_inf, neg_inf};   // token g + 8 (e >> 1), head 2tq + (e & 1)
      if (!ti.bad) {
        float sp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint32_t kaddr = ring_addr + slot * L::kKBytes + warp * L::kHeadBytes;
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
          s4[e] = (!head_valid[e & 1] || tk >= ti.ntok) ? neg_inf : v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);   // the key rows are no longer needed
      if (++slot == NS) { slot = 0; phase ^= 1u; }

      const int js = (ti.t0 % kDecTile) / kDhChunk;   // stage of the tile (splits start on a tile)
#pragma unroll
      for (int j = 0; j < TS; ++j)
        if (j == js) {
#pragma unroll
          for (int e = 0; e < 4; ++e) st[j][e] = s4[e];
          t_ntok |= uint32_t(ti.bad ? 0 : ti.ntok) << (5 * j);
          if (lane == 0) note[j] = ti.page;
        }
      const bool last = (ti.flags & 2) != 0;
      if (js != TS - 1 && !last) continue;

      // ---- the tile is scored: first a finished split's pending P V (its last V rows had this tile's K
      // stream to land) and its result
      if (fin_pending) {
        while (vq_n > 0 && ok) ok = pv_oldest();
        if (!ok) break;
        write_split(note[4], note[5], note[6], note[7]);
        fin_pending = false;
      }

      // ---- decision: row maxima of the tile against the split's running maximum
      const int seq = ti.seq, grp = ti.grp;
      const int t_t0 = ti.t0 - js * kDhChunk;   // the tile's first token
      float T[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v = neg_inf;
#pragma unroll
        for (int j = 0; j < TS; ++j)
          if (j <= js) v = fmaxf(v, fmaxf(st[j][c], st[j][c + 2]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        T[c] = v;
      }
      bool keep[2];
      {
        // the rule for one row: no visible score in the tile, or a finite running maximum that the
        // tile stays below by more than -log2(lambda)
        bool row_ok[2];
#pragma unroll
        for (int c = 0; c < 2; ++c)
          row_ok[c] = !head_valid[c] || T[c] == neg_inf || (m_run[c] != neg_inf && (T[c] - m_run[c]) < p.log2_lambda);
        const int tile = t_t0 / kDecTile;
        if constexpr (PER_HEAD) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            keep[c] = head_valid[c] && !(active && row_ok[c]);
            if (g == 0 && head_valid[c]) {
              if (p.skip_mask) {
                const int hq = (grp * HG + warp) * G + 2 * tq + c;
                p.skip_mask[(size_t(seq) * p.Hq + hq) * p.max_tiles + tile] = keep[c] ? 0 : 1;
              }
              n_skipped += keep[c] ? 0 : 1;
            }
          }
        } else {
          const bool unit_skip = active && __all_sync(0xffffffffu, row_ok[0] && row_ok[1]);
          keep[0] = head_valid[0] && !unit_skip;
          keep[1] = head_valid[1] && !unit_skip;
          if (lane == 0) {
            if (p.skip_mask)
              p.skip_mask[(size_t(seq) * p.Hkv + grp * HG + warp) * p.max_tiles + tile] = unit_skip ? 1 : 0;
            n_skipped += unit_skip ? 1 : 0;
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) m_run[c] = fmaxf(m_run[c], T[c]);   // a dropped tile lies below it anyway
      }

      if (__any_sync(0xffffffffu, keep[0] || keep[1])) {
        // ---- ask for the tile's V rows of this KV head, in the buffer after the pending ones (the
        // oldest tile's P V first when every buffer is taken)
        if (vq_n == NB && !pv_oldest()) { ok = false; break; }
        const int b = vq_head + vq_n < NB ? vq_head + vq_n : vq_head + vq_n - NB;
        if (lane == 0) {
          uint32_t bytes = 0;
#pragma unroll
          for (int j = 0; j < TS; ++j)
            if (j <= js && ((t_ntok >> (5 * j)) & 31u)) bytes += uint32_t(L::kHeadBytes);
          fence_proxy_async_smem();   // the buffer's previous rows were read (ldmatrix) before this write
          mbar_arrive_expect_tx(&my_vfull[b], bytes);
#pragma unroll
          for (int j = 0; j < TS; ++j)
            if (j <= js && ((t_ntok >> (5 * j)) & 31u))
              tma_load_5d(vbuf + b * L::kVWarp + j * L::kHeadBytes, &tm_v, &my_vfull[b], 0,
                          (t_t0 + j * kDhChunk) % p.page_size, 0, grp * HG + warp, note[j]);
        }
        // ---- raise the reference past the threshold (the pending tiles' P V first: their P was taken
        // against the old reference), then the tile's P^T (skipped heads contribute nothing)
        float alpha[2] = {1.f, 1.f};
        bool raised = false;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float mx = keep[c] ? T[c] : neg_inf;
          if (mx != neg_inf && (m_ref[c] == neg_inf || mx > m_ref[c] + kDecRescaleThreshold)) {
            alpha[c] = (m_ref[c] == neg_inf) ? 0.f : fast_exp2(m_ref[c] - mx);
            m_ref[c] = mx;
            raised = true;
          }
        }
        if (__any_sync(0xffffffffu, raised)) {
          while (vq_n > 0 && ok) ok = pv_oldest();
          if (!ok) {
            ++vq_n;   // the copy just asked for (buffer b, after the pending ones) is drained below too
            break;
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            o[m][0] *= alpha[0]; o[m][2] *= alpha[0];
            o[m][1] *= alpha[1]; o[m][3] *= alpha[1];
          }
          l_part[0] *= alpha[0]; lr_part[0] *= alpha[0];
          l_part[1] *= alpha[1]; lr_part[1] *= alpha[1];
        }
        const float off[2] = {m_ref[0] == neg_inf ? 0.f : m_ref[0], m_ref[1] == neg_inf ? 0.f : m_ref[1]};
        uint32_t pt[TS][2];
#pragma unroll
        for (int j = 0; j < TS; ++j) {
          pt[j][0] = pt[j][1] = 0u;
          if (j > js) continue;
          float pr[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[e] = keep[e & 1] ? fast_exp2(st[j][e] - off[e & 1]) : 0.f;
          l_part[0] += pr[0] + pr[2];
          l_part[1] += pr[1] + pr[3];
          // the weights applied to V are normalised by the sum of the rounded P
          const uint32_t x0 = pack_bf16x2(pr[0], pr[1]);   // token g, heads 2tq, 2tq + 1
          const uint32_t x1 = pack_bf16x2(pr[2], pr[3]);   // token g + 8
          lr_part[0] += bf16_lo(x0) + bf16_lo(x1);
          lr_part[1] += bf16_hi(x0) + bf16_hi(x1);
          pt[j][0] = movmatrix_trans(x0);
          pt[j][1] = movmatrix_trans(x1);
        }
#pragma unroll
        for (int bb = 0; bb < NB; ++bb)
          if (bb == b) {
#pragma unroll
            for (int j = 0; j < TS; ++j) {
              pb[bb][j][0] = pt[j][0];
              pb[bb][j][1] = pt[j][1];
            }
            pv_ntok[bb] = t_ntok;
          }
        ++vq_n;
      }
      t_ntok = 0;
#pragma unroll
      for (int j = 0; j < TS; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[j][e] = neg_inf;
      if (!last) continue;

      // ---- the split's end: its result follows at the next tile's end (or the CTA's), once its last
      // tiles' V rows have landed
      if (lane == 0) {
        note[4] = seq; note[5] = grp; note[6] = ti.split;
        note[7] = (ti.len + p.split_tokens - 1) / p.split_tokens;
      }
      __syncwarp();
      fin_pending = true;
    }
    if (ok && fin_pending) {   // the CTA's last split
      while (vq_n > 0 && ok) ok = pv_oldest();
      if (ok) write_split(note[4], note[5], note[6], note[7]);
    }
    // copies of this warp still in flight land before the CTA exits
    if (lane == 0)
      for (int i = 0, b = vq_head; i < vq_n; ++i, b = b + 1 == NB ? 0 : b + 1)
        mbar_drain(&my_vfull[b], (v_phase >> b) & 1u);
    if (p.skipped_tiles) {
      uint32_t n = n_skipped;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) n += __shfl_xor_sync(0xffffffffu, n, d);
      if (lane == 0 && n) atomicAdd(p.skipped_tiles, (unsigned long long)n);
    }
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace attn
