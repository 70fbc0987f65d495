// Tiled prefill attention for sm_100a: TMA-staged K/V tiles, tcgen05 MMAs with
// fp32 accumulators in tensor memory, online softmax in registers.
//
// A persistent CTA walks work items (b, hq, 256-row query block), longest
// causal blocks first. The query block is two 128-row tiles, A and B, that
// share every K/V tile the CTA loads. Roles (384 threads):
//   warp 0      TMA producer: Q_A, Q_B once per item, then K_0, K_1, V_0,
//               K_2, V_1, ... into a ring (each K one tile ahead of its V)
//   warps 1, 2  MMA issuers, one thread per query tile; warp 1 owns the TMEM allocation
//   warps 4-7   softmax of tile A (thread t <-> row t <-> TMEM lane t)
//   warps 8-11  softmax of tile B
// Tensor memory (512 columns): S_A | S_B | O_A | O_B, fp32.
// Per KV tile j the issuer of tile X issues S_X(j+1) = Q_X K_{j+1}^T as soon as
// the softmax of tile X has copied S_X(j) into registers, and O_X += P_X(j) V_j
// once the softmax has written the bf16 probabilities P_X(j) to shared
// memory; the two tiles' issuers never wait on each other's softmax. So the exponentials of tile j overlap the next tile's Q K^T, and
// the tensor pipe has queued work while either softmax warpgroup computes.
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
// setmaxnreg split: warps 0-3 drop to 96 registers, warps 4-11 rise to 200.
constexpr int kPfRegsLow = 96, kPfRegsHigh = 200;
constexpr int kPfRegPoolNeeded = 128 * kPfRegsLow + 256 * kPfRegsHigh;  // must fit the launch allocation

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
                       bTeardown = 14, bKVFull = 15, bKVEmpty = 15 + kStages, kNumBars = 15 + 2 * kStages;
  static constexpr int kMisc = kBars + 8 * kNumBars;            // tmem base, flags, votes
  static constexpr int kTotal = kMisc + 256;
  static constexpr int kDynamic = kTotal + 1024;
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
template <int D>
__device__ __forceinline__ void pf_issue_pv(uint32_t d_tmem, uint64_t pdesc, uint64_t vdesc, bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kPfKeys / 16; ++kk) {
    const uint64_t poff16 = uint64_t(((kk / 4) * (kPfRows * 128) + (kk % 4) * 32) >> 4);
    umma_ss(d_tmem, pdesc + poff16, vdesc + uint64_t((kk * 16 * 128) >> 4), idesc,
            (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool CAUSAL, bool SKIP>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NS = L::kStages;
  constexpr int kTmemCols = 512;

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
      mbar_init(&bars[L::bSFree + x], 4);    // one arrival per softmax warp
      mbar_init(&bars[L::bPFull + x], 4);
      mbar_init(&bars[L::bPVDone + x], 1);
      mbar_init(&bars[L::bOEmpty + x], 4);
    }
    mbar_init(&bars[L::bTeardown], 2);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars[L::bKVFull + s], 1);
      mbar_init(&bars[L::bKVEmpty + s], 2);   // both MMA issuers release each slot
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

  // Register split (launch: 168 x 384 = 64512): warps 0-3 keep kPfRegsLow = 96, the two
  // softmax warpgroups take kPfRegsHigh = 200 each: 128*96 + 256*200 = 63488 <= 64512.
  if (warp < 4) {
    setmaxnreg_dec<kPfRegsLow>();
    if (warp == 0) {
      // ============================================================ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t qe_bits = 3u;
        uint32_t pend_mask = 0, pend_ph = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
          int qb, b, hq;
          item_coords(item, qb, b, hq);
          const int kvh = hq / (p.Hq / p.Hkv);
          const int rows0 = tile_rows(qb, 0), rows1 = tile_rows(qb, 1);
          const int n = max(tile_nkv(qb, 0, rows0), tile_nkv(qb, 1, rows1));
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if ((x == 0 ? rows0 : rows1) == 0 || !ok) continue;
            if (!mbar_wait(&bars[L::bQEmpty + x], (qe_bits >> x) & 1u, abort_flag, p.status)) { ok = false; continue; }
            qe_bits ^= 1u << x;
            mbar_arrive_expect_tx(&bars[L::bQFull + x], L::kTileBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + L::kQ + x * L::kTileBytes + c * L::kChunkBytes, &tm_q, &bars[L::bQFull + x],
                          c * 64, qb * 2 * kPfRows + x * kPfRows, hq, b);
          }
          // K_0, then K_{j+1} before V_j: the order in which the MMA thread consumes them
          for (int step = 0; step < 2 * n && ok; ++step) {
            // step 0: K_0; step 2j+1: K_{j+1} (or V_j when j is the last tile); step 2j+2: V_j
            const int j = (step - 1) / 2;
            const bool is_k = step == 0 || (step % 2 == 1 && j + 1 < n);
            const int key0 = step == 0 ? 0 : (is_k ? (j + 1) * kPfKeys : (step % 2 == 1 ? j : step / 2 - 1) * kPfKeys);
            if (!mbar_wait(&bars[L::bKVEmpty + slot], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars[L::bKVFull + slot], L::kTileBytes);
            const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + L::kRing + slot * L::kTileBytes + c * L::kChunkBytes, tm, &bars[L::bKVFull + slot],
                          c * 64, key0, kvh, b);
            pend_mask |= 1u << slot;
            pend_ph = (pend_ph & ~(1u << slot)) | (phase << slot);
            if (++slot == NS) { slot = 0; phase ^= 1u; }
          }
        }
        if (!ok) {
          for (int s = 0; s < NS; ++s)
            if (pend_mask & (1u << s)) mbar_drain(&bars[L::bKVFull + s], (pend_ph >> s) & 1u);
        }
      }
    } else if (warp == 1 || warp == 2) {
      // ============================================================ MMA issuers
      // One thread per query tile x (warp 1: A, warp 2: B). Both walk the whole
      // K/V ring of every item and arrive on each slot's empty barrier (count 2),
      // whether or not their tile uses the slot; an issuer never runs more than
      // one ring phase ahead because it waits for each slot's load first.
      if (lane == 0) {
        const int x = warp - 1;
        const uint32_t q_desc_addr = smem_u32(smem + L::kQ + x * L::kTileBytes);
        const uint32_t p_desc_addr = smem_u32(smem + L::kP + x * L::kPBytes);
        const uint32_t ring_addr = smem_u32(smem + L::kRing);
        const uint32_t d_s = tmem + pf_col_s(x), d_o = tmem + pf_col_o<D>(x);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t qf_ph = 0u, sfree_ph = 0u, pf_ph = 0u, oe_ph = 1u;
        bool qk_started = false;  // a Q K^T has been issued for this tile in this kernel
        bool ok = true;

        for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
          int qb, b, hq;
          item_coords(item, qb, b, hq);
          const int rows0 = tile_rows(qb, 0), rows1 = tile_rows(qb, 1);
          const int n = max(tile_nkv(qb, 0, rows0), tile_nkv(qb, 1, rows1));
          const int nkv = tile_nkv(qb, x, x == 0 ? rows0 : rows1);
          if (nkv > 0) {
            if (!mbar_wait(&bars[L::bQFull + x], qf_ph, abort_flag, p.status)) break;
            qf_ph ^= 1u;
          }
          bool pv_started = false;  // a P V product was issued for this tile in this item
          // ring uses of the item, in order: K_0, then K_{j+1} (if any) and V_j for each j
          for (int step = 0; step < 2 * n && ok; ++step) {
            const int j = (step - 1) / 2;
            const bool is_k = step == 0 || (step % 2 == 1 && j + 1 < n);
            const int tile = step == 0 ? 0 : (is_k ? j + 1 : (step % 2 == 1 ? j : step / 2 - 1));
            const int cur = slot;
            const uint32_t cph = phase;
            if (++slot == NS) { slot = 0; phase ^= 1u; }
            if (!mbar_wait(&bars[L::bKVFull + cur], cph, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            if (is_k && tile < nkv) {
              // S_x(tile) = Q_x K_tile^T, once the softmax has copied out S_x(tile - 1)
              if (qk_started) {
                if (!mbar_wait(&bars[L::bSFree + x], sfree_ph, abort_flag, p.status)) { ok = false; break; }
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
              if (!mbar_wait(&bars[L::bPFull + x], pf_ph, abort_flag, p.status)) { ok = false; break; }
              pf_ph ^= 1u;
              tc_fence_after();
              const bool skip_pv = SKIP && pv_skip[x] != 0;
              if (!skip_pv) {
                if (!pv_started) {
                  // first P V of this item: the previous item's epilogue must have read O_x
                  if (!mbar_wait(&bars[L::bOEmpty + x], oe_ph, abort_flag, p.status)) { ok = false; break; }
                  oe_ph ^= 1u;
                  tc_fence_after();
                }
                pf_issue_pv<D>(d_o, make_sdesc_sw128(p_desc_addr, 16, 1024),
                               make_sdesc_sw128(ring_addr + cur * L::kTileBytes, L::kChunkBytes, 1024), pv_started);
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
    int own_timeout_only = 0;
    volatile int* no_abort = reinterpret_cast<volatile int*>(&own_timeout_only);
    uint32_t sf_ph = 0, pvd_ph = 0;
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
        uint32_t sr[kPfKeys];
        ATTN_TMEM_LD32_NOWAIT(taddr_s + 0, sr + 0);
        ATTN_TMEM_LD32_NOWAIT(taddr_s + 32, sr + 32);
        ATTN_TMEM_LD32_NOWAIT(taddr_s + 64, sr + 64);
        ATTN_TMEM_LD32_NOWAIT(taddr_s + 96, sr + 96);
        tmem_ld_wait();
        ATTN_REG_FENCE32(sr + 0);
        ATTN_REG_FENCE32(sr + 32);
        ATTN_REG_FENCE32(sr + 64);
        ATTN_REG_FENCE32(sr + 96);
        // S_x is in registers: the tensor pipe may overwrite it with the next tile
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::bSFree + x]);

        float s[kPfKeys];
#pragma unroll
        for (int e = 0; e < kPfKeys; ++e) s[e] = __uint_as_float(sr[e]);
        const int key0 = j * kPfKeys;
        const bool full_tile = (!CAUSAL || key0 + kPfKeys - 1 <= row0) && (key0 + kPfKeys <= p.S);
        if (!full_tile) {
#pragma unroll
          for (int e = 0; e < kPfKeys; ++e) {
            const int key = key0 + e;
            if ((CAUSAL && key > row) || key >= p.S) s[e] = neg_inf;
          }
        }
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
        uint32_t pk[kPfKeys / 2];   // this row's probabilities, bf16 pairs
        float alpha = 1.f;
        bool raise = false;
        if (!skip_all) {
          float m_tile = neg_inf;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (!skip_h[h]) m_tile = fmaxf(m_tile, r2[h]);
          // raise the reference maximum only when needed (or on the first finite tile)
          raise = (m_tile != neg_inf) && (m_ref == neg_inf || m_tile > m_ref + kRescaleThreshold);
          if (raise) {
            alpha = (m_ref == neg_inf) ? 0.f : fast_exp2(m_ref - m_tile);
            m_ref = m_tile;
            l *= alpha;
          }
          const float offset = (m_ref == neg_inf) ? 0.f : m_ref;
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t negoff2 = f2_pack(-offset, -offset);
          uint64_t sum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int e = 0; e < kPfKeys / 2; ++e) {
            if (skip_h[e / 32]) {
              pk[e] = 0u;
            } else {
              const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), scale2, negoff2);
              float x0, x1;
              f2_unpack(xx, x0, x1);
              const float p0 = fast_exp2(x0);
              const float p1 = fast_exp2(x1);
              sum2[e & 1] = f2_add(sum2[e & 1], f2_pack(p0, p1));
              pk[e] = pack_bf16x2(p0, p1);
            }
          }
          float sa, sb, sc, sd;
          f2_unpack(sum2[0], sa, sb);
          f2_unpack(sum2[1], sc, sd);
          l += (sa + sb) + (sc + sd);
        }
        // P_x(j-1) must have been consumed (and O_x updated) before P_x(j) is written
        // and before any rescale of O_x; the exponentials above overlapped that P V.
        if (j > 0) {
          if (!mbar_wait(&bars[L::bPVDone + x], pvd_ph, no_abort, p.status)) { ok = false; break; }
          pvd_ph ^= 1u;
          tc_fence_after();
        }
        if (!skip_all) {
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
        if (t == 0) pv_skip[x] = skip_all ? 1 : 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::bPFull + x]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait(&bars[L::bPVDone + x], pvd_ph, no_abort, p.status)) { ok = false; break; }
      pvd_ph ^= 1u;
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bOEmpty + x]);
    }
  }

  __syncwarp();  // reconverge the producer and MMA warps (one lane worked)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
