// Dense paged decode with one CTA item per group of KV heads.
//
// Work item = (split, sequence, group of HG KV heads), handed out in that
// order (largest splits first) by an atomic ticket counter in the workspace,
// which the host zeroes before the launch; when the grid has a CTA for every
// item, CTA b takes item b and the counter is not used. A stage is 16 tokens of the item:
// one TMA copy brings the K rows of all HG heads (a contiguous 16-token x HG-head
// block of a page) and one the V rows; the tensor map orders heads outside
// tokens, so each head's 16 rows land as one 4 KB (D = 128) 128-byte-swizzled
// block. The producer warp reads the next item's length and first block-table
// window one item ahead and ships each item's query rows with its first stage.
//
// Consumer warp h owns KV head h of the group: per stage it computes its G query
// heads' scores for the 16 tokens and P.V with mma.m16n8k16 (rows >= G zero),
// runs the online softmax in its accumulator registers across the whole item,
// and writes the item's result for its heads at the end -- no cross-warp merge.
// Split partials are combined by decode_merge_kernel as in the per-head path.
//
// F8 = true reads a cache stored as FP8 E4M3 codes with one scale per pool
// (K = k_scale * code, V = v_scale * code; k_scale is folded into the score
// scale and v_scale into the output normalisation on the host). A head's 16
// tokens are then one 2 KB block of 128-byte rows (D = 128). The codes go from
// shared memory straight into mma fragments, widened to f16 on the way (exact),
// and the query rows are taken to f16 once per item:
//   * q K^T: the head dimension is summed over, so it may be visited in any
//     order that q and K share. Lane (g, t) loads bytes [32t, 32t + 32) of key
//     row g; in k-step ks its fragment halves hold bytes 32t + 4ks + {0, 1} and
//     32t + 4ks + {2, 3}, and its q fragments take the same dimensions.
//   * P V: output column c of n-tile n is head dimension 16c + n, so lane
//     (g, t) loads byte group g (dims 16g .. 16g + 15) of the token rows it
//     needs, pairs the bytes of two tokens with a byte permute, and ends up
//     owning output dims 32t .. 32t + 31 (o[n][0] = dim 32t + n,
//     o[n][1] = dim 32t + 16 + n).
// P is rounded to f16 for P V and the normaliser sums the rounded values.
#pragma once

#include "decode.cuh"

namespace attn {

constexpr int kDhChunk = 16;  // tokens per TMA copy (one 16-slot block of a page)

// For G <= 8 the consumers run the transposed products (below) with groups of
// 4 KV heads and several CTAs per SM, fewer stages each: three 5-warp CTAs
// (two for G = 8) keep 12 consumer warps resident, which hide each other's
// latency. The FP8 cache also doubles the stage to 32 tokens (two copies per
// tensor) to spread the per-stage costs over more tokens.
constexpr int kTrBlocks = 3;   // resident CTAs per SM for G <= 4 (registers: 3 x 160 threads x <= 136)

// BLOCKS = 0: the default residency below; BLOCKS = 2 serves grids of at most two items per
// SM (a single long sequence), whose CTAs then keep three stages in flight instead of two.
template <int D, int G, int HG, bool F8 = false, int BLOCKS = 0>
struct DecodeHeadsSmem {
  static constexpr bool kTr = G <= 8;                            // transposed products
  static constexpr int kHalves = (kTr && F8) ? 2 : 1;            // 16-token copies per tensor per stage
  static constexpr int kTok = kDhChunk * kHalves;                // tokens per stage
  static constexpr int kBlocks = BLOCKS > 0 ? BLOCKS : (kTr ? (G <= 4 ? kTrBlocks : 2) : 1);   // CTAs per SM
  static constexpr int kHeadBytes = kDhChunk * D * (F8 ? 1 : 2);   // one head's 16 tokens
  static constexpr int kHalfBytes = HG * kHeadBytes;             // one copy: 16 tokens of the HG heads
  static constexpr int kKVBytes = kHalves * kHalfBytes;          // K (or V) rows of one stage
  static constexpr int kQBytes = HG * G * D * 2;        // the item's query rows
  static constexpr int kStageBytes = (2 * kKVBytes + kQBytes + 1023) / 1024 * 1024;
  static constexpr int kFit = (233472 / kBlocks - 1024 - 2048) / (kStageBytes + 48);
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kFull = kRing;
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kInfo = kEmpty + 8 * kStages;   // TileInfo per stage
  static constexpr int kTotal = kInfo + 32 * kStages;
  static constexpr int kDynamic = kTotal + 1024;
  static_assert(kDynamic <= 232448, "shared memory per block");
  static_assert(kStages >= 2, "ring depth");
};

// Byte offset of 16-byte chunk `c` (0 .. D/8 - 1) of token `t` (0 .. 15) in one head's
// bf16 block of a stage. The copy orders the block [64-column half][token][64 columns]:
// 128-byte row (c / 8) * 16 + t, unit (c mod 8) XOR t mod 8, so eight consecutive
// tokens of one half sit in eight different bank groups.
template <int D>
__device__ __forceinline__ uint32_t dh_swz(int t, int c) {
  const int row = (c >> 3) * kDhChunk + t;
  return uint32_t(row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// item -> (split, seq, group): splits outermost so that full-length splits go first
__device__ __forceinline__ void dh_item_coords(long long item, int num_seqs, int n_groups, int& seq, int& split,
                                               int& grp) {
  const long long per = (long long)num_seqs * n_groups;
  split = int(item / per);
  const int rem = int(item % per);
  seq = rem / n_groups;
  grp = rem % n_groups;
}

template <int D, int G, int HG, bool F8 = false, int BLOCKS = 0>
__global__ void __launch_bounds__((HG + 1) * 32, DecodeHeadsSmem<D, G, HG, F8, BLOCKS>::kBlocks)
    decode_heads_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p, int* ticket_counter) {
  static_assert(G >= 1 && G <= 16, "query heads per KV head");
  static_assert(!F8 || D == 128, "the FP8 cache layout assumes 128-byte rows");
  using L = DecodeHeadsSmem<D, G, HG, F8, BLOCKS>;
  launch_dependents();   // let the merge kernel be scheduled early; it waits for this grid to finish
  constexpr int NS = L::kStages;
  constexpr int KS = D / 16;
  constexpr int NT = D / 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + L::kInfo);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;
  const int n_groups = p.Hkv / HG;
  const long long num_items = (long long)p.max_splits * p.num_seqs * n_groups;

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
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    int slot = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pending_phase = 0;
    bool ok = true;
    // next item (ticket), its length and first block-table window, one item ahead
    long long nx_item = 0;
    int nx_len = 0, nx_win = -1;
    bool first_fetch = true;
    auto fetch_next = [&]() {
      long long t = 0;
      if (p.static_items) {
        t = first_fetch ? (long long)blockIdx.x : num_items;
      } else {
        if (lane == 0) t = atomicAdd(ticket_counter, 1);
        t = __shfl_sync(0xffffffffu, t, 0);
      }
      first_fetch = false;
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
      for (int t0 = t_begin; t0 < t_end && ok; t0 += L::kTok) {
        const int e0 = t0 / p.page_size;
        if ((e0 >> 5) != win) {   // a stage advances by at most two pages, so by at most one window
          win = e0 >> 5;
          win_cur = win_next;
          const int e = (win + 1) * 32 + lane;
          win_next = e < p.max_pages ? __ldg(&bt_row[e]) : -1;
        }
        if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        // the page of each 16-token copy (the second may sit on the next page, even in the next window)
        int page[L::kHalves];
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h) {
          const int e = (t0 + h * kDhChunk) / p.page_size;
          page[h] = __shfl_sync(0xffffffffu, (e >> 5) == win ? win_cur : win_next, e & 31);
        }
        if (lane == 0) {
          const bool first = t0 == t_begin;
          TileInfo ti;
          ti.seq = seq; ti.split = split; ti.kvh = grp; ti.t0 = t0;
          ti.ntok = min(L::kTok, len - t0);
          ti.bad = 0;
          uint32_t bytes = first ? uint32_t(L::kQBytes) : 0u;
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h) {
            if (h * kDhChunk >= ti.ntok) { ti.bad |= 1 << h; continue; }   // past the end: not copied
            if (page[h] >= 0 && page[h] < p.num_pages) {
              bytes += uint32_t(2 * L::kHalfBytes);
            } else {
              raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
              ti.bad |= 1 << h;
            }
          }
          ti.flags = (first ? 1 : 0) | (t0 + L::kTok >= t_end ? 2 : 0);
          ti.len = len;
          info[slot] = ti;
          uint8_t* stage = smem + slot * L::kStageBytes;
          mbar_arrive_expect_tx(&full[slot], bytes);
          if (first) bulk_load(stage + 2 * L::kKVBytes, qsrc, uint32_t(L::kQBytes), &full[slot]);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h) {
            if (ti.bad & (1 << h)) continue;
            const int in_page = (t0 + h * kDhChunk) % p.page_size;
            uint8_t* kdst = stage + h * L::kHalfBytes;
            if constexpr (F8) {
              tma_load_4d(kdst, &tm_k, &full[slot], 0, in_page, grp * HG, page[h]);
              tma_load_4d(kdst + L::kKVBytes, &tm_v, &full[slot], 0, in_page, grp * HG, page[h]);
            } else {
              tma_load_5d(kdst, &tm_k, &full[slot], 0, in_page, 0, grp * HG, page[h]);
              tma_load_5d(kdst + L::kKVBytes, &tm_v, &full[slot], 0, in_page, 0, grp * HG, page[h]);
            }
          }
        }
        __syncwarp();
        pending |= 1u << slot;
        pending_phase = (pending_phase & ~(1u << slot)) | (phase << slot);
        if (++slot == NS) { slot = 0; phase ^= 1u; }
      }
    }
    if (ok && mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) {
      if (lane == 0) {  // end-of-work marker: a stage with no copies
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
  } else if constexpr (L::kTr) {
    // ------------------------------------------------------------ consumer warp, G <= 8: transposed products
    // S^T = K q^T (tokens on the 16-row side, query heads on the 8 columns) and O^T = V^T P^T, so that
    // one mma covers 16 tokens x G heads: half the mma, exp2 and accumulator count of the q-on-rows
    // form. Lane (g, t): S^T rows (tokens) g and g + 8, columns (heads) 2t and 2t + 1. P^T goes from
    // the S^T accumulator layout to the P^T operand layout with one 8x8 transpose per 8 tokens.
    // O^T m-tile m, row r is head dim 16m + r for bf16 (operands from ldmatrix), and 16r + m (r < 8),
    // 16(r - 8) + 8 + m (r >= 8) for FP8, where lane (g, t) then holds dims 16g .. 16g + 15.
    const float neg_inf = -__int_as_float(0x7f800000);
    const int g = lane >> 2, tq = lane & 3;
    const bool head_valid[2] = {2 * tq < G, 2 * tq + 1 < G};
    int slot = 0;
    uint32_t phase = 0;
    int no_abort = 0;
    bool ok = true;
    int seq = 0, split = 0, grp = 0, n_splits = 0;
    constexpr int MT = D / 16;   // m-tiles of O^T
    uint32_t qb[KS][2];
    float o[MT][4];
    const uint32_t ring_addr = smem_u32(smem);
    float m_ref[2] = {neg_inf, neg_inf};   // heads 2tq, 2tq + 1
    float l_part[2] = {0.f, 0.f};
    float lr_part[2] = {0.f, 0.f};

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) { ok = false; break; }
      const TileInfo ti = info[slot];
      if (ti.flags & 4) break;
      uint8_t* stage = smem + slot * L::kStageBytes;
      if (ti.flags & 1) {
        seq = ti.seq; split = ti.split; grp = ti.kvh;
        n_splits = (ti.len + p.split_tokens - 1) / p.split_tokens;
        // q^T operand: column g = query head g of this KV head; FP8: dims 32tq + 4ks + {0,1} / {2,3}
        // (matching the key fragments), bf16: dims 16ks + 2tq + {0,1} / + 8
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(stage + 2 * L::kKVBytes) + warp * G * (D / 2);
        const bool qv = g < G;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          if constexpr (F8) {
            qb[ks][0] = qv ? bf16x2_to_f16x2(qs[g * (D / 2) + 16 * tq + 2 * ks]) : 0u;
            qb[ks][1] = qv ? bf16x2_to_f16x2(qs[g * (D / 2) + 16 * tq + 2 * ks + 1]) : 0u;
          } else {
            qb[ks][0] = qv ? qs[g * (D / 2) + ks * 8 + tq] : 0u;
            qb[ks][1] = qv ? qs[g * (D / 2) + ks * 8 + 4 + tq] : 0u;
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        m_ref[0] = m_ref[1] = neg_inf;
        l_part[0] = l_part[1] = 0.f;
        lr_part[0] = lr_part[1] = 0.f;
      }
      const bool last = (ti.flags & 2) != 0;
      if (ti.bad != (1 << L::kHalves) - 1) {
        const int ntok = ti.ntok;
        const int bad = ti.bad;
        // ---- S^T = K q^T per 16-token half: key rows g and g + 8 (swizzle phase g), bytes [32tq, 32tq + 32)
        float st[L::kHalves][4];
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h) {
          float sp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          if constexpr (F8) {
            const uint8_t* kb = stage + h * L::kHalfBytes + warp * L::kHeadBytes;
            const uint4 r0a = *reinterpret_cast<const uint4*>(kb + g * 128 + (((2 * tq) ^ g) << 4));
            const uint4 r0b = *reinterpret_cast<const uint4*>(kb + g * 128 + (((2 * tq + 1) ^ g) << 4));
            const uint4 r1a = *reinterpret_cast<const uint4*>(kb + (g + 8) * 128 + (((2 * tq) ^ g) << 4));
            const uint4 r1b = *reinterpret_cast<const uint4*>(kb + (g + 8) * 128 + (((2 * tq + 1) ^ g) << 4));
            const uint32_t w0[8] = {r0a.x, r0a.y, r0a.z, r0a.w, r0b.x, r0b.y, r0b.z, r0b.w};
            const uint32_t w1[8] = {r1a.x, r1a.y, r1a.z, r1a.w, r1b.x, r1b.y, r1b.z, r1b.w};
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              uint32_t a[4];
              e4m3x4_to_f16x2x2(w0[ks], a[0], a[2]);
              e4m3x4_to_f16x2x2(w1[ks], a[1], a[3]);
              mma_f16_16816(sp[ks & 1], a, qb[ks][0], qb[ks][1]);
            }
          } else {
            // K operand by ldmatrix: matrix mi = tokens 8 (mi & 1) .., dims 16ks + 8 (mi >> 1) ..
            const uint32_t kaddr = ring_addr + slot * L::kStageBytes + h * L::kHalfBytes + warp * L::kHeadBytes;
            const int mi = lane >> 3, r = lane & 7;
            const int tok = (mi & 1) * 8 + r;
            uint32_t af[KS][4];
#pragma unroll
            for (int ks = 0; ks < KS; ++ks)
              ldsm_x4(kaddr + dh_swz<D>(tok, ks * 2 + (mi >> 1)), af[ks][0], af[ks][1], af[ks][2], af[ks][3]);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) mma_bf16_16816(sp[ks & 1], af[ks], qb[ks][0], qb[ks][1]);
          }
          // st[h][e]: token 16h + g + 8 (e >> 1), head 2tq + (e & 1); half h not copied -> all masked
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = h * kDhChunk + g + 8 * (e >> 1);
            const float v = (sp[0][e] + sp[1][e]) * p.scale_log2;
            st[h][e] = (!head_valid[e & 1] || tok >= ntok || ((bad >> h) & 1)) ? neg_inf : v;
          }
        }
        float mx[2] = {fmaxf(st[0][0], st[0][2]), fmaxf(st[0][1], st[0][3])};
#pragma unroll
        for (int h = 1; h < L::kHalves; ++h) {
          mx[0] = fmaxf(mx[0], fmaxf(st[h][0], st[h][2]));
          mx[1] = fmaxf(mx[1], fmaxf(st[h][1], st[h][3]));
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 4));
          mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 8));
          mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 16));
        }
        float alpha[2] = {1.f, 1.f};
        bool raised = false;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (mx[c] != neg_inf && (m_ref[c] == neg_inf || mx[c] > m_ref[c] + kDecRescaleThreshold)) {
            alpha[c] = (m_ref[c] == neg_inf) ? 0.f : fast_exp2(m_ref[c] - mx[c]);
            m_ref[c] = mx[c];
            raised = true;
          }
        }
        if (__any_sync(0xffffffffu, raised)) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            o[m][0] *= alpha[0]; o[m][2] *= alpha[0];
            o[m][1] *= alpha[1]; o[m][3] *= alpha[1];
          }
          l_part[0] *= alpha[0]; lr_part[0] *= alpha[0];
          l_part[1] *= alpha[1]; lr_part[1] *= alpha[1];
        }
        uint32_t pb[L::kHalves][2];   // P^T operand per half: tokens 2tq, 2tq + 1 (and + 8) of head g
        {
          const float off[2] = {m_ref[0] == neg_inf ? 0.f : m_ref[0], m_ref[1] == neg_inf ? 0.f : m_ref[1]};
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h) {
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(st[h][e] - off[e & 1]);
            l_part[0] += pr[0] + pr[2];
            l_part[1] += pr[1] + pr[3];
            // the weights applied to V are normalised by the sum of the rounded P
            uint32_t x0, x1;   // tokens g and g + 8, heads 2tq, 2tq + 1
            if constexpr (F8) {
              x0 = pack_f16x2(pr[0], pr[1]);
              x1 = pack_f16x2(pr[2], pr[3]);
              lr_part[0] += f16_lo(x0) + f16_lo(x1);
              lr_part[1] += f16_hi(x0) + f16_hi(x1);
            } else {
              x0 = pack_bf16x2(pr[0], pr[1]);
              x1 = pack_bf16x2(pr[2], pr[3]);
              lr_part[0] += bf16_lo(x0) + bf16_lo(x1);
              lr_part[1] += bf16_hi(x0) + bf16_hi(x1);
            }
            pb[h][0] = movmatrix_trans(x0);
            pb[h][1] = movmatrix_trans(x1);
          }
        }
        // ---- O^T += V^T P^T per half: token rows 2tq, 2tq + 1, 2tq + 8, 2tq + 9, byte group g (dims 16g ..);
        // rows past the end or of a half not copied are zeroed so that 0 * (stale or NaN) cannot reach O
        if constexpr (!F8) {
          // V^T operand by transposing ldmatrix: matrix mi = tokens 8 (mi >> 1) .., dims 16m + 8 (mi & 1) ..;
          // a[0], a[1] hold tokens 2tq, 2tq + 1 and a[2], a[3] tokens 2tq + 8, 2tq + 9 (low, high half)
          const uint32_t vaddr = ring_addr + slot * L::kStageBytes + L::kKVBytes + warp * L::kHeadBytes;
          const int mi = lane >> 3, r = lane & 7;
          const int tok = (mi >> 1) * 8 + r;
          const uint32_t mk0 = (2 * tq < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 1 < ntok ? 0xFFFF0000u : 0u);
          const uint32_t mk1 = (2 * tq + 8 < ntok ? 0x0000FFFFu : 0u) | (2 * tq + 9 < ntok ? 0xFFFF0000u : 0u);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            uint32_t a[4];
            ldsm_x4_t(vaddr + dh_swz<D>(tok, 2 * m + (mi & 1)), a[0], a[1], a[2], a[3]);
            a[0] &= mk0; a[1] &= mk0; a[2] &= mk1; a[3] &= mk1;
            mma_bf16_16816(o[m], a, pb[0][0], pb[0][1]);
          }
        }
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h) {
          if (!F8 || ((bad >> h) & 1)) continue;
          const uint8_t* vb = stage + L::kKVBytes + h * L::kHalfBytes + warp * L::kHeadBytes;
          uint4 vr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tok = 2 * tq + (i & 1) + (i >> 1) * 8;
            vr[i] = *reinterpret_cast<const uint4*>(vb + tok * 128 + ((g ^ (tok & 7)) << 4));
            if (h * kDhChunk + tok >= ntok) vr[i] = make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            // m-tiles 4w .. 4w + 3: rows g (dim 16g + m, word w) and g + 8 (dim 16g + 8 + m, word w + 2)
            uint32_t a0[4], a1[4], a2[4], a3[4];
            const uint32_t A0 = (&vr[0].x)[w], B0 = (&vr[1].x)[w], C0 = (&vr[2].x)[w], D0 = (&vr[3].x)[w];
            const uint32_t A1 = (&vr[0].x)[w + 2], B1 = (&vr[1].x)[w + 2], C1 = (&vr[2].x)[w + 2],
                           D1 = (&vr[3].x)[w + 2];
            e4m3x4_to_f16x2x2(__byte_perm(A0, B0, 0x5140), a0[0], a0[1]);
            e4m3x4_to_f16x2x2(__byte_perm(A0, B0, 0x7362), a0[2], a0[3]);
            e4m3x4_to_f16x2x2(__byte_perm(A1, B1, 0x5140), a1[0], a1[1]);
            e4m3x4_to_f16x2x2(__byte_perm(A1, B1, 0x7362), a1[2], a1[3]);
            e4m3x4_to_f16x2x2(__byte_perm(C0, D0, 0x5140), a2[0], a2[1]);
            e4m3x4_to_f16x2x2(__byte_perm(C0, D0, 0x7362), a2[2], a2[3]);
            e4m3x4_to_f16x2x2(__byte_perm(C1, D1, 0x5140), a3[0], a3[1]);
            e4m3x4_to_f16x2x2(__byte_perm(C1, D1, 0x7362), a3[2], a3[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t a[4] = {a0[i], a1[i], a2[i], a3[i]};
              mma_f16_16816(o[4 * w + i], a, pb[h][0], pb[h][1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == NS) { slot = 0; phase ^= 1u; }
      if (!last) continue;

      // ---- the item's result for heads 2tq, 2tq + 1 of this warp's KV head
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
        const int hq = (grp * HG + warp) * G + 2 * tq + c;
        const float lsum = l_part[c];
        float inv = lr_part[c] > 0.f ? 1.f / lr_part[c] : 0.f;   // 0 only if every page was invalid
        if constexpr (F8) inv *= p.v_scale;
        if (n_splits == 1) {
          if constexpr (F8) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + (size_t(seq) * p.Hq + hq) * D + 16 * g);
            dst[0] = make_uint4(pack_bf16x2(o[0][c] * inv, o[1][c] * inv), pack_bf16x2(o[2][c] * inv, o[3][c] * inv),
                                pack_bf16x2(o[4][c] * inv, o[5][c] * inv), pack_bf16x2(o[6][c] * inv, o[7][c] * inv));
            dst[1] = make_uint4(pack_bf16x2(o[0][c + 2] * inv, o[1][c + 2] * inv),
                                pack_bf16x2(o[2][c + 2] * inv, o[3][c + 2] * inv),
                                pack_bf16x2(o[4][c + 2] * inv, o[5][c + 2] * inv),
                                pack_bf16x2(o[6][c + 2] * inv, o[7][c + 2] * inv));
          } else {
            __nv_bfloat16* dst = p.o + (size_t(seq) * p.Hq + hq) * D + g;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              dst[16 * m] = __float2bfloat16_rn(o[m][c] * inv);
              dst[16 * m + 8] = __float2bfloat16_rn(o[m][c + 2] * inv);
            }
          }
          if (p.lse && g == 0)
            p.lse[size_t(seq) * p.Hq + hq] = lsum > 0.f ? (m_ref[c] + __log2f(lsum)) * 0.69314718055994531f : neg_inf;
        } else {
          const uint64_t keep = l2_keep_policy();   // the merge reads these back after the KV stream
          if constexpr (F8) {
            float* dst = p.ws_o + ((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + 16 * g;
            st_keep(dst, o[0][c] * inv, o[1][c] * inv, o[2][c] * inv, o[3][c] * inv, keep);
            st_keep(dst + 4, o[4][c] * inv, o[5][c] * inv, o[6][c] * inv, o[7][c] * inv, keep);
            st_keep(dst + 8, o[0][c + 2] * inv, o[1][c + 2] * inv, o[2][c + 2] * inv, o[3][c + 2] * inv, keep);
            st_keep(dst + 12, o[4][c + 2] * inv, o[5][c + 2] * inv, o[6][c + 2] * inv, o[7][c + 2] * inv, keep);
          } else {
            float* dst = p.ws_o + ((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + g;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              st_keep(dst + 16 * m, o[m][c] * inv, keep);
              st_keep(dst + 16 * m + 8, o[m][c + 2] * inv, keep);
            }
          }
          if (g == 0)
            st_keep(&p.ws_lse[(size_t(seq) * p.max_splits + split) * p.Hq + hq],
                    lsum > 0.f ? m_ref[c] + __log2f(lsum) : neg_inf, keep);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumer warp = KV head `warp` of the group
    const float neg_inf = -__int_as_float(0x7f800000);
    const int g = lane >> 2, tq = lane & 3;
    const bool row0_valid = g < G, row1_valid = g + 8 < G;
    int slot = 0;
    uint32_t phase = 0;
    int no_abort = 0;
    bool ok = true;
    const uint32_t ring_addr = smem_u32(smem);
    int seq = 0, split = 0, grp = 0, n_splits = 0;
    uint32_t qa[KS][4];
    float o[NT][4];
    float m_ref[2] = {neg_inf, neg_inf};
    float l_part[2] = {0.f, 0.f};    // row sums of the probabilities (-> LSE)
    float lr_part[2] = {0.f, 0.f};   // the same as rounded to bf16 for P V (-> normalises O)

    while (ok) {
      if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) { ok = false; break; }
      const TileInfo ti = info[slot];
      if (ti.flags & 4) break;
      uint8_t* stage = smem + slot * L::kStageBytes;
      if (ti.flags & 1) {
        seq = ti.seq; split = ti.split; grp = ti.kvh;
        n_splits = (ti.len + p.split_tokens - 1) / p.split_tokens;
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(stage + 2 * L::kKVBytes) + warp * G * (D / 2);
        const int h0 = row0_valid ? g : 0, h1 = row1_valid ? g + 8 : 0;
        if constexpr (F8) {
          // dims 32tq + 4ks + {0,1} and {2,3}, matching the key fragments below
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            qa[ks][0] = row0_valid ? bf16x2_to_f16x2(qs[h0 * (D / 2) + 16 * tq + 2 * ks]) : 0u;
            qa[ks][1] = row1_valid ? bf16x2_to_f16x2(qs[h1 * (D / 2) + 16 * tq + 2 * ks]) : 0u;
            qa[ks][2] = row0_valid ? bf16x2_to_f16x2(qs[h0 * (D / 2) + 16 * tq + 2 * ks + 1]) : 0u;
            qa[ks][3] = row1_valid ? bf16x2_to_f16x2(qs[h1 * (D / 2) + 16 * tq + 2 * ks + 1]) : 0u;
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            qa[ks][0] = row0_valid ? qs[h0 * (D / 2) + ks * 8 + tq] : 0u;
            qa[ks][1] = row1_valid ? qs[h1 * (D / 2) + ks * 8 + tq] : 0u;
            qa[ks][2] = row0_valid ? qs[h0 * (D / 2) + ks * 8 + 4 + tq] : 0u;
            qa[ks][3] = row1_valid ? qs[h1 * (D / 2) + ks * 8 + 4 + tq] : 0u;
          }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m_ref[0] = m_ref[1] = neg_inf;
        l_part[0] = l_part[1] = 0.f;
        lr_part[0] = lr_part[1] = 0.f;
      }
      const bool last = (ti.flags & 2) != 0;
      if (!ti.bad) {
        const int ntok = ti.ntok;
        const uint32_t kaddr = ring_addr + slot * L::kStageBytes + warp * L::kHeadBytes;
        const uint32_t vaddr = kaddr + L::kKVBytes;
        // ---- S = q K^T (16 tokens = two 8-token column tiles; k-steps alternate accumulators)
        float s[2][4];
        {
          float sp[2][2][4];
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int a = 0; a < 2; ++a) sp[j][a][0] = sp[j][a][1] = sp[j][a][2] = sp[j][a][3] = 0.f;
          if constexpr (F8) {
            // key row j*8 + g (its swizzle phase is g), bytes [32tq, 32tq + 32)
            const uint8_t* kb = stage + warp * L::kHeadBytes;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint8_t* row = kb + (j * 8 + g) * 128;
              const uint4 w0 = *reinterpret_cast<const uint4*>(row + (((2 * tq) ^ g) << 4));
              const uint4 w1 = *reinterpret_cast<const uint4*>(row + (((2 * tq + 1) ^ g) << 4));
              const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
              for (int ks = 0; ks < KS; ++ks) {
                uint32_t b0, b1;
                e4m3x4_to_f16x2x2(w[ks], b0, b1);
                mma_f16_16816(sp[j][ks & 1], qa[ks], b0, b1);
              }
            }
          } else {
            const int mi = lane >> 3, r = lane & 7;
            const int tok = (mi >> 1) * 8 + r;
            uint32_t bfr[KS][4];
#pragma unroll
            for (int ks = 0; ks < KS; ++ks)
              ldsm_x4(kaddr + dh_swz<D>(tok, ks * 2 + (mi & 1)), bfr[ks][0], bfr[ks][1], bfr[ks][2], bfr[ks][3]);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              mma_bf16_16816(sp[0][ks & 1], qa[ks], bfr[ks][0], bfr[ks][1]);
              mma_bf16_16816(sp[1][ks & 1], qa[ks], bfr[ks][2], bfr[ks][3]);
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[j][e] = sp[j][0][e] + sp[j][1][e];
        }
        const bool clean = ntok == kDhChunk;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = j * 8 + 2 * tq + (e & 1);
            const float v = s[j][e] * p.scale_log2;
            s[j][e] = (!clean && tok >= ntok) ? neg_inf : v;
          }
        float mx[2];
        mx[0] = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        mx[1] = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        }
        if (!F8 && !clean) {
          // zero the V rows of tokens past the end so that 0 * (stale or NaN) cannot reach O
          for (int t = ntok; t < kDhChunk; ++t)
            for (int c = lane; c < D / 8; c += 32)
              *reinterpret_cast<uint4*>(stage + L::kKVBytes + warp * L::kHeadBytes + dh_swz<D>(t, c)) =
                  make_uint4(0, 0, 0, 0);
          __syncwarp();
        }
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
        uint32_t pa[4];
        {
          const float off0 = m_ref[0] == neg_inf ? 0.f : m_ref[0];
          const float off1 = m_ref[1] == neg_inf ? 0.f : m_ref[1];
          float pr[2][4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            pr[j][0] = row0_valid ? fast_exp2(s[j][0] - off0) : 0.f;
            pr[j][1] = row0_valid ? fast_exp2(s[j][1] - off0) : 0.f;
            pr[j][2] = row1_valid ? fast_exp2(s[j][2] - off1) : 0.f;
            pr[j][3] = row1_valid ? fast_exp2(s[j][3] - off1) : 0.f;
          }
          l_part[0] += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
          l_part[1] += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
          // the weights applied to V are normalised by the sum of the rounded P, so
          // they add up to one (a dominant key's P, up to 2^8 under the lagging
          // reference, would otherwise carry its rounding into the whole row)
          if constexpr (F8) {
            pa[0] = pack_f16x2(pr[0][0], pr[0][1]);
            pa[1] = pack_f16x2(pr[0][2], pr[0][3]);
            pa[2] = pack_f16x2(pr[1][0], pr[1][1]);
            pa[3] = pack_f16x2(pr[1][2], pr[1][3]);
            lr_part[0] += (f16_lo(pa[0]) + f16_hi(pa[0])) + (f16_lo(pa[2]) + f16_hi(pa[2]));
            lr_part[1] += (f16_lo(pa[1]) + f16_hi(pa[1])) + (f16_lo(pa[3]) + f16_hi(pa[3]));
          } else {
            pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
            pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
            pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
            pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
            lr_part[0] += (bf16_lo(pa[0]) + bf16_hi(pa[0])) + (bf16_lo(pa[2]) + bf16_hi(pa[2]));
            lr_part[1] += (bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3]));
          }
        }
        // ---- O += P V over the 16 tokens
        if constexpr (F8) {
          // token rows 2tq, 2tq + 1, 2tq + 8, 2tq + 9 (swizzle phases 2tq, 2tq + 1), byte group g;
          // rows past the end are zeroed here so that 0 * (stale or NaN) cannot reach O
          const uint8_t* vb = stage + L::kKVBytes + warp * L::kHeadBytes;
          uint4 vr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tok = 2 * tq + (i & 1) + (i >> 1) * 8;
            vr[i] = *reinterpret_cast<const uint4*>(vb + tok * 128 + ((g ^ (tok & 7)) << 4));
            if (!clean && tok >= ntok) vr[i] = make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t a = (&vr[0].x)[w], b = (&vr[1].x)[w], c = (&vr[2].x)[w], d = (&vr[3].x)[w];
            uint32_t b0[4], b1[4];   // n-tile 4w + i: (token 2tq, 2tq + 1) and (2tq + 8, 2tq + 9)
            e4m3x4_to_f16x2x2(__byte_perm(a, b, 0x5140), b0[0], b0[1]);
            e4m3x4_to_f16x2x2(__byte_perm(a, b, 0x7362), b0[2], b0[3]);
            e4m3x4_to_f16x2x2(__byte_perm(c, d, 0x5140), b1[0], b1[1]);
            e4m3x4_to_f16x2x2(__byte_perm(c, d, 0x7362), b1[2], b1[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i) mma_f16_16816(o[4 * w + i], pa, b0[i], b1[i]);
          }
        } else {
          const int mi = lane >> 3, r = lane & 7;
          const int tok = (mi & 1) * 8 + r;
#pragma unroll
          for (int n2 = 0; n2 < NT / 2; ++n2) {
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(vaddr + dh_swz<D>(tok, n2 * 2 + (mi >> 1)), v0, v1, v2, v3);
            mma_bf16_16816(o[2 * n2], pa, v0, v1);
            mma_bf16_16816(o[2 * n2 + 1], pa, v2, v3);
          }
        }
        if (!F8 && !clean) fence_proxy_async_smem();   // zeroed rows before the next TMA write
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == NS) { slot = 0; phase ^= 1u; }
      if (!last) continue;

      // ---- the item's result for this warp's G query heads
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 1);
        l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 2);
        lr_part[r] += __shfl_xor_sync(0xffffffffu, lr_part[r], 1);
        lr_part[r] += __shfl_xor_sync(0xffffffffu, lr_part[r], 2);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const bool valid = r == 0 ? row0_valid : row1_valid;
        if (!valid) continue;
        const int hq = (grp * HG + warp) * G + g + 8 * r;
        const float lsum = l_part[r];
        float inv = lr_part[r] > 0.f ? 1.f / lr_part[r] : 0.f;   // 0 only if every page was invalid
        if constexpr (F8) inv *= p.v_scale;
        if (n_splits == 1) {
          if constexpr (F8) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + (size_t(seq) * p.Hq + hq) * D + 32 * tq);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int q8 = 0; q8 < 2; ++q8) {
                const int n = 8 * q8, e = 2 * r + h;
                dst[2 * h + q8] = make_uint4(pack_bf16x2(o[n][e] * inv, o[n + 1][e] * inv),
                                             pack_bf16x2(o[n + 2][e] * inv, o[n + 3][e] * inv),
                                             pack_bf16x2(o[n + 4][e] * inv, o[n + 5][e] * inv),
                                             pack_bf16x2(o[n + 6][e] * inv, o[n + 7][e] * inv));
              }
          } else {
            __nv_bfloat16* dst = p.o + (size_t(seq) * p.Hq + hq) * D + 2 * tq;
#pragma unroll
            for (int n = 0; n < NT; ++n)
              *reinterpret_cast<uint32_t*>(dst + n * 8) = pack_bf16x2(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
          }
          if (p.lse && tq == 0)
            p.lse[size_t(seq) * p.Hq + hq] = lsum > 0.f ? (m_ref[r] + __log2f(lsum)) * 0.69314718055994531f : neg_inf;
        } else {
          const uint64_t keep = l2_keep_policy();   // the merge reads these back after the KV stream
          if constexpr (F8) {
            float* dst = p.ws_o + ((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + 32 * tq;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int n = 0; n < NT; n += 4) {
                const int e = 2 * r + h;
                st_keep(dst + 16 * h + n, o[n][e] * inv, o[n + 1][e] * inv, o[n + 2][e] * inv, o[n + 3][e] * inv,
                        keep);
              }
          } else {
            float* dst = p.ws_o + ((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + 2 * tq;
#pragma unroll
            for (int n = 0; n < NT; ++n) st_keep(dst + n * 8, o[n][2 * r] * inv, o[n][2 * r + 1] * inv, keep);
          }
          if (tq == 0)
            st_keep(&p.ws_lse[(size_t(seq) * p.max_splits + split) * p.Hq + hq],
                    lsum > 0.f ? m_ref[r] + __log2f(lsum) : neg_inf, keep);
        }
      }
    }
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace attn
