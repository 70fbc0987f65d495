// Tiled prefill attention for sm_100a: TMA-staged K/V tiles, tcgen05 MMAs with
// fp32 accumulators in tensor memory, online softmax in registers.
//
// A persistent CTA walks work items (b, hq, 256-row query block), longest
// causal blocks first. The query block is two 128-row tiles, A and B, that
// share every K/V tile the CTA loads. Roles (384 threads):
//   warp 0      TMA producer: Q_A, Q_B once per item, then K_j, V_j into a ring
//   warp 1      MMA issuer (one thread): S_X = Q_X K_j^T into TMEM, then
//               O_X += P_X V_j with P_X read from TMEM; owns the TMEM allocation
//   warps 4-7   softmax of tile A (thread t <-> row t <-> TMEM lane t)
//   warps 8-11  softmax of tile B
// Tensor memory (512 columns): S_A | S_B | O_A | O_B. P_X (bf16, two per
// column) overwrites the first half of S_X once S_X is in registers.
// MMA issue order per KV tile j: PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1), so
// softmax A of tile j+1 overlaps the tensor core working on B, and vice versa.
// The exponentials use a reference maximum that is only raised when the tile
// maximum exceeds it by more than 2^8 (exact: O and l share the reference);
// the BLASST decisions use the true running maximum of the kept tiles.
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
  long long num_items;
  float scale_log2;    // scale * log2(e)
  float log2_lambda;   // log2(lambda) (tile skip only)
};

constexpr int kPfRows = 128;     // rows per query tile
constexpr int kPfKeys = 128;     // keys per K/V tile (two 64-key decision tiles)
constexpr int kPfThreads = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct PrefillSmem {
  static constexpr int kTileBytes = kPfRows * D * 2;            // one Q, K or V tile
  static constexpr int kChunkBytes = kPfRows * 128;             // 64 columns x 128 rows, SW128
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kQ = 0;                                  // Q_A, Q_B
  static constexpr int kRing = 2 * kTileBytes;
  static constexpr int kBars = kRing + kStages * kTileBytes;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 2, bSFull = 4, bPFull = 6, bOFull = 8, bOEmpty = 10,
                       bTeardown = 12, bKVFull = 13, bKVEmpty = 13 + kStages, kNumBars = 13 + 2 * kStages;
  static constexpr int kMisc = kBars + 8 * kNumBars;            // tmem base, flags, votes
  static constexpr int kTotal = kMisc + 256;
  static constexpr int kDynamic = kTotal + 1024;
};

template <int D, bool CAUSAL, bool SKIP>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NS = L::kStages;
  constexpr int kTmemCols = 512;
  constexpr uint32_t kColS[2] = {0, 128};
  constexpr uint32_t kColO[2] = {256, 256 + D};

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* pv_skip = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);      // [2]
  volatile int* votes = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);       // [2][4 warps][4]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars[L::bQFull + x], 1);
      mbar_init(&bars[L::bQEmpty + x], 1);
      mbar_init(&bars[L::bSFull + x], 1);
      mbar_init(&bars[L::bPFull + x], kPfRows);
      mbar_init(&bars[L::bOFull + x], 1);
      mbar_init(&bars[L::bOEmpty + x], kPfRows);
    }
    mbar_init(&bars[L::bTeardown], 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars[L::bKVFull + s], 1);
      mbar_init(&bars[L::bKVEmpty + s], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  // Item decode shared by all roles: longest causal blocks first; the G query
  // heads of one KV head are adjacent so their K/V tiles are reused from L2.
  auto item_coords = [&](long long item, int& qb, int& b, int& hq) {
    const long long per = (long long)p.B * p.Hq;
    qb = p.n_qblocks - 1 - int(item / per);
    const int rem = int(item % per);
    b = rem / p.Hq;
    hq = rem % p.Hq;
  };
  auto tile_rows = [&](int qb, int x) { return max(0, min(kPfRows, p.S - qb * 2 * kPfRows - x * kPfRows)); };
  auto tile_nkv = [&](int qb, int x, int rows) {
    if (rows == 0) return 0;
    if (CAUSAL) return (qb * 2 * kPfRows + x * kPfRows + rows - 1) / kPfKeys + 1;
    return (p.S + kPfKeys - 1) / kPfKeys;
  };

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int slot = 0;
      uint32_t phase = 0;
      uint32_t qe_ph[2] = {1u, 1u};
      uint32_t pend_mask = 0, pend_ph = 0;
      bool ok = true;
      for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
        int qb, b, hq;
        item_coords(item, qb, b, hq);
        const int kvh = hq / (p.Hq / p.Hkv);
        int rows[2], nkv[2];
        for (int x = 0; x < 2; ++x) { rows[x] = tile_rows(qb, x); nkv[x] = tile_nkv(qb, x, rows[x]); }
        const int n = max(nkv[0], nkv[1]);
        for (int x = 0; x < 2 && ok; ++x) {
          if (rows[x] == 0) continue;
          if (!mbar_wait(&bars[L::bQEmpty + x], qe_ph[x], abort_flag, p.status)) { ok = false; break; }
          qe_ph[x] ^= 1u;
          mbar_arrive_expect_tx(&bars[L::bQFull + x], L::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(smem + L::kQ + x * L::kTileBytes + c * L::kChunkBytes, &tm_q, &bars[L::bQFull + x],
                        c * 64, qb * 2 * kPfRows + x * kPfRows, hq, b);
        }
        for (int j = 0; j < n && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {  // K_j then V_j
            if (!mbar_wait(&bars[L::bKVEmpty + slot], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars[L::bKVFull + slot], L::kTileBytes);
            const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + L::kRing + slot * L::kTileBytes + c * L::kChunkBytes, tm,
                          &bars[L::bKVFull + slot], c * 64, j * kPfKeys, kvh, b);
            pend_mask |= 1u << slot;
            pend_ph = (pend_ph & ~(1u << slot)) | (phase << slot);
            if (++slot == NS) { slot = 0; phase ^= 1u; }
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < NS; ++s)
          if (pend_mask & (1u << s)) mbar_drain(&bars[L::bKVFull + s], (pend_ph >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, kPfKeys, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t ring_addr = smem_u32(smem + L::kRing);
      int slot = 0;
      uint32_t phase = 0;
      uint32_t qf_ph[2] = {0u, 0u}, pf_ph[2] = {0u, 0u}, oe_ph[2] = {1u, 1u};
      bool ok = true;

      auto issue_qk = [&](int x, int kslot) {
        const uint32_t qa = q_addr + x * L::kTileBytes;
        const uint32_t ka = ring_addr + kslot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::kChunkBytes + (kk % 4) * 32;
          umma_ss(tmem + kColS[x], make_sdesc_sw128(qa + off, 16, 1024), make_sdesc_sw128(ka + off, 16, 1024),
                  idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int x, int vslot, bool accumulate) {
        const uint32_t va = ring_addr + vslot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kPfKeys / 16; ++kk) {
          umma_ts(tmem + kColO[x], tmem + kColS[x] + kk * 8,
                  make_sdesc_sw128(va + kk * 16 * 128, L::kChunkBytes, 1024), idesc_pv,
                  (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      auto next_slot = [&](int& s, uint32_t& ph) {
        const int cur = s;
        if (++s == NS) { s = 0; ph ^= 1u; }
        return cur;
      };

      for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
        int qb, b, hq;
        item_coords(item, qb, b, hq);
        int rows[2], nkv[2];
        for (int x = 0; x < 2; ++x) { rows[x] = tile_rows(qb, x); nkv[x] = tile_nkv(qb, x, rows[x]); }
        const int n = max(nkv[0], nkv[1]);
        for (int x = 0; x < 2 && ok; ++x) {
          if (rows[x] == 0) continue;
          ok = mbar_wait(&bars[L::bQFull + x], qf_ph[x], abort_flag, p.status);
          qf_ph[x] ^= 1u;
        }
        if (!ok) break;
        // K_0
        uint32_t kph = phase;
        int kslot = next_slot(slot, phase);
        if (!mbar_wait(&bars[L::bKVFull + kslot], kph, abort_flag, p.status)) break;
        tc_fence_after();
        for (int x = 0; x < 2; ++x) {
          if (nkv[x] == 0) continue;
          issue_qk(x, kslot);
          umma_commit(&bars[L::bSFull + x]);
        }
        umma_commit(&bars[L::bKVEmpty + kslot]);
        bool pv_started[2] = {false, false};
        bool first_pv[2] = {true, true};
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t vph = phase;
          const int vslot = next_slot(slot, phase);
          if (!mbar_wait(&bars[L::bKVFull + vslot], vph, abort_flag, p.status)) { ok = false; break; }
          const bool has_next = j + 1 < n;
          uint32_t nph = 0;
          int nslot = -1;
          bool next_ready = false;
          if (has_next) { nph = phase; nslot = next_slot(slot, phase); }
          for (int x = 0; x < 2 && ok; ++x) {
            if (j >= nkv[x]) continue;
            if (!mbar_wait(&bars[L::bPFull + x], pf_ph[x], abort_flag, p.status)) { ok = false; break; }
            pf_ph[x] ^= 1u;
            tc_fence_after();
            const bool skip_pv = SKIP && pv_skip[x] != 0;
            if (!skip_pv) {
              if (first_pv[x]) {
                if (!mbar_wait(&bars[L::bOEmpty + x], oe_ph[x], abort_flag, p.status)) { ok = false; break; }
                oe_ph[x] ^= 1u;
                first_pv[x] = false;
                tc_fence_after();
              }
              issue_pv(x, vslot, pv_started[x]);
              pv_started[x] = true;
            }
            if (j + 1 < nkv[x]) {
              if (!next_ready) {
                if (!mbar_wait(&bars[L::bKVFull + nslot], nph, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                next_ready = true;
              }
              issue_qk(x, nslot);
              umma_commit(&bars[L::bSFull + x]);
            } else {
              umma_commit(&bars[L::bOFull + x]);
              umma_commit(&bars[L::bQEmpty + x]);
            }
          }
          if (!ok) break;
          if (has_next) umma_commit(&bars[L::bKVEmpty + nslot]);
          umma_commit(&bars[L::bKVEmpty + vslot]);
        }
      }
      // every MMA issued so far must finish before the TMEM is released
      umma_commit(&bars[L::bTeardown]);
      mbar_drain(&bars[L::bTeardown], 0);
    }
  } else if (warp >= 4) {
    // ============================================================ softmax warpgroups
    const int x = (warp - 4) / 4;          // 0: tile A, 1: tile B
    const int wq = warp & 3;               // TMEM lane quadrant
    const int t = wq * 32 + lane;          // row within the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t taddr_s = tmem + lane_off + kColS[x];
    const uint32_t taddr_o = tmem + lane_off + kColO[x];
    const float neg_inf = -__int_as_float(0x7f800000);
    int own_timeout_only = 0;
    volatile int* no_abort = reinterpret_cast<volatile int*>(&own_timeout_only);
    uint32_t sf_ph = 0, of_ph = 0;
    bool ok = true;

    for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      int qb, b, hq;
      item_coords(item, qb, b, hq);
      const int rows = tile_rows(qb, x);
      const int nkv = tile_nkv(qb, x, rows);
      if (nkv == 0) continue;
      const int row0 = qb * 2 * kPfRows + x * kPfRows;
      const int row = row0 + t;
      const bool row_valid = t < rows;
      const int last_row = row0 + rows - 1;
      float m_ref = neg_inf, m_true = neg_inf, l = 0.f;

      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&bars[L::bSFull + x], sf_ph, no_abort, p.status)) { ok = false; break; }
        sf_ph ^= 1u;
        tc_fence_after();
        float s[kPfKeys];
#pragma unroll
        for (int c = 0; c < kPfKeys / 32; ++c) {
          uint32_t r[32];
          ATTN_TMEM_LD32(taddr_s + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
        }
        const int key0 = j * kPfKeys;
        const bool full_tile = (!CAUSAL || key0 + kPfKeys - 1 <= row0) && (key0 + kPfKeys <= p.S);
        if (!full_tile) {
#pragma unroll
          for (int e = 0; e < kPfKeys; ++e) {
            const int key = key0 + e;
            if ((CAUSAL && key > row) || key >= p.S) s[e] = neg_inf;
          }
        }
        float mx[2] = {neg_inf, neg_inf};
#pragma unroll
        for (int e = 0; e < kPfKeys; ++e) mx[e / 64] = fmaxf(mx[e / 64], s[e]);
        float r2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) r2[h] = (mx[h] == neg_inf) ? neg_inf : mx[h] * p.scale_log2;

        bool skip_h[2] = {false, false};
        if constexpr (SKIP) {
          // Decisions for both 64-key halves with one barrier: half 1 is voted
          // under both outcomes of half 0.
          auto row_ok = [&](float r, float m) {
            return !row_valid || r == neg_inf || (m != neg_inf && (r - m) < p.log2_lambda);
          };
          const bool ok0 = row_ok(r2[0], m_true);
          const bool ok1_if_skip0 = row_ok(r2[1], m_true);
          const bool ok1_if_keep0 = row_ok(r2[1], fmaxf(m_true, r2[0]));
          const int v0 = __all_sync(0xffffffffu, ok0);
          const int v1 = __all_sync(0xffffffffu, ok1_if_skip0);
          const int v2 = __all_sync(0xffffffffu, ok1_if_keep0);
          volatile int* my_votes = votes + (x * 4 + wq) * 4;
          if (lane == 0) { my_votes[0] = v0; my_votes[1] = v1; my_votes[2] = v2; }
          named_bar_sync(1 + x, 128);
          int a0 = 1, a1 = 1, a2 = 1;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            a0 &= votes[(x * 4 + w) * 4 + 0];
            a1 &= votes[(x * 4 + w) * 4 + 1];
            a2 &= votes[(x * 4 + w) * 4 + 2];
          }
          skip_h[0] = a0 != 0;
          skip_h[1] = skip_h[0] ? (a1 != 0) : (a2 != 0);
          if (!skip_h[0]) m_true = fmaxf(m_true, r2[0]);
          if (!skip_h[1]) m_true = fmaxf(m_true, r2[1]);
          if (p.skip_mask && t == 0) {
            const int qt = qb * 2 + x;
            uint8_t* mrow = p.skip_mask + ((size_t(b) * p.Hq + hq) * p.n_qt + qt) * p.n_kt;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int k64 = key0 + h * 64;
              const bool visited = k64 < p.S && (!CAUSAL || k64 <= last_row);
              if (visited) mrow[k64 / 64] = skip_h[h] ? 1 : 0;
            }
          }
        }
        const bool skip_all = skip_h[0] && skip_h[1];
        if (!skip_all) {
          float m_tile = neg_inf;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (!skip_h[h]) m_tile = fmaxf(m_tile, r2[h]);
          // raise the reference maximum only when needed (or on the first finite tile)
          const bool raise = (m_tile != neg_inf) && (m_ref == neg_inf || m_tile > m_ref + kRescaleThreshold);
          float alpha = 1.f;
          if (raise) {
            alpha = (m_ref == neg_inf) ? 0.f : fast_exp2(m_ref - m_tile);
            m_ref = m_tile;
            l *= alpha;
          }
          if (__any_sync(0xffffffffu, raise && j > 0)) {
            // rescale this warp's rows of O (PV of tile j-1 finished before S_j was committed)
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              ATTN_TMEM_LD32(taddr_o + c * 32, r);
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              ATTN_TMEM_ST32(taddr_o + c * 32, r);
            }
          }
          const float offset = (m_ref == neg_inf) ? 0.f : m_ref;
          float rowsum = 0.f;
#pragma unroll
          for (int c = 0; c < kPfKeys / 32; ++c) {
            uint32_t pk[16];
            const bool zero_chunk = skip_h[c / 2];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float p0 = 0.f, p1 = 0.f;
              if (!zero_chunk) {
                p0 = fast_exp2(fmaf(s[c * 32 + 2 * e], p.scale_log2, -offset));
                p1 = fast_exp2(fmaf(s[c * 32 + 2 * e + 1], p.scale_log2, -offset));
              }
              rowsum += p0 + p1;
              pk[e] = pack_bf16x2(p0, p1);
            }
            ATTN_TMEM_ST16(taddr_s + c * 16, pk);
          }
          l += rowsum;
          tmem_st_wait();
        }
        tc_fence_before();
        if (t == 0) pv_skip[x] = skip_all ? 1 : 0;
        mbar_arrive(&bars[L::bPFull + x]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait(&bars[L::bOFull + x], of_ph, no_abort, p.status)) { ok = false; break; }
      of_ph ^= 1u;
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
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
            (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : neg_inf;
      tc_fence_before();
      mbar_arrive(&bars[L::bOEmpty + x]);
    }
  }

  __syncwarp();  // reconverge the producer and MMA warps (one lane worked)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
