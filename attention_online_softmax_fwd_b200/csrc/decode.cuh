// Paged single-token decode: split-KV attention kernel + log-sum-exp merge.
//
// Work item = (sequence, split, KV head). A persistent CTA walks its items in
// a strided order. One producer warp streams the item's 64-token tiles of K
// and V from the page pool into a shared-memory ring with TMA copies, one copy
// per (page chunk, K|V), addressed through the block table. Eight consumer
// warps each take 8 tokens of a tile and all G query heads of the KV head:
// lanes split the head dimension for q.k (partial dots reduced with a
// butterfly reduce-scatter) and for P.V. The softmax state (running max m,
// sum l, accumulator O) follows the online recurrence over the split's tiles;
// m is shared by the eight warps (one named barrier per tile), l and O are
// per warp and summed at the end of the item. A split's result is written as a
// partial (O / l, log2-sum-exp); the merge kernel combines the splits.
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
  uint8_t* skip_mask;          // [N][Hkv][max_tiles] or null
  int* status;                 // caller's device status word or null
  int num_seqs, Hq, Hkv, page_size, max_pages, num_pages;
  int split_tokens, max_splits, max_tiles;
  int chunk;          // tokens per TMA copy: min(page_size, 64)
  float scale_log2;   // softmax scale * log2(e)
  float log2_lambda;  // log2(lambda) for the tile skip
  long long num_items;
};

constexpr int kDecTile = 64;          // tokens per tile (= BLASST decision tile)
constexpr int kDecConsumerWarps = 8;  // 8 tokens of each tile per warp
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecStages = 4;

template <int D, int G>
struct DecodeSmem {
  static constexpr int kStageBytes = 2 * kDecTile * D * 2;  // K and V tiles, bf16
  static constexpr int kRing = kDecStages * kStageBytes;
  // offsets (bytes) from the 1024-aligned base
  static constexpr int kFull = kRing;
  static constexpr int kEmpty = kFull + 8 * kDecStages;
  static constexpr int kInfo = kEmpty + 8 * kDecStages;                  // int2 per stage
  static constexpr int kScore = kInfo + 8 * kDecStages;                  // [warps][8*G] floats
  static constexpr int kRed = kScore + 4 * kDecConsumerWarps * 8 * G;    // [2][warps][G] floats
  static constexpr int kCombL = kRed + 4 * 2 * kDecConsumerWarps * G;    // [2][G] floats
  static constexpr int kCombO = (kCombL + 4 * 2 * G + 15) / 16 * 16;     // [G][D] floats
  static constexpr int kTotal = kCombO + 4 * G * D;
  static constexpr int kDynamic = kTotal + 1024;                         // slack for alignment
};

__device__ __forceinline__ void decode_item_coords(long long item, int Hkv, int max_splits, int& seq, int& split,
                                                   int& kvh) {
  kvh = int(item % Hkv);
  long long rest = item / Hkv;
  split = int(rest % max_splits);
  seq = int(rest / max_splits);
}

// Load the D/32 consecutive bf16 of one row that belong to `lane`, as fp32.
template <int D>
__device__ __forceinline__ void load_row_slice(const __nv_bfloat16* row, int lane, float (&x)[D / 32]) {
  if constexpr (D == 128) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + lane * 4);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + lane * 2);
    x[0] = bf16_lo(w); x[1] = bf16_hi(w);
  }
}

template <int D, int G, bool SKIP>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p) {
  using L = DecodeSmem<D, G>;
  constexpr int DL = D / 32;                              // head dims per lane
  constexpr int TB = (G >= 4) ? (32 / G < 1 ? 1 : 32 / G) : 8;  // tokens per reduce batch
  constexpr int TBc = TB > 8 ? 8 : TB;
  constexpr int NB = 8 / TBc;                             // reduce batches per tile
  constexpr int V = TBc * G;                              // values per batch (<= 32)
  constexpr int DUP = 32 / V;                             // lanes holding the same value

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::kEmpty);
  int2* info = reinterpret_cast<int2*>(smem + L::kInfo);
  float* score = reinterpret_cast<float*>(smem + L::kScore);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* comb_l = reinterpret_cast<float*>(smem + L::kCombL);
  float* comb_o = reinterpret_cast<float*>(smem + L::kCombO);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int capacity = p.max_pages * p.page_size;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumerWarps);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) comb_o[i] = 0.f;
  for (int i = threadIdx.x; i < 2 * G; i += blockDim.x) comb_l[i] = 0.f;
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const int nchunks = kDecTile / p.chunk;
    const uint32_t chunk_bytes = uint32_t(p.chunk) * D * 2;
    int slot = 0;
    uint32_t phase = 0;
    uint32_t pending = 0;  // stages with copies issued, for the abort path
    uint32_t pending_phase = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      int seq, split, kvh;
      decode_item_coords(item, p.Hkv, p.max_splits, seq, split, kvh);
      int len = __ldg(&p.seq_lens[seq]);
      if (len > capacity || len < 0) {
        if (lane == 0 && split == 0 && kvh == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
        len = len < 0 ? 0 : capacity;
      }
      const int t_begin = split * p.split_tokens;
      if (t_begin >= len) continue;
      const int t_end = min(t_begin + p.split_tokens, len);
      const int32_t* bt_row = p.block_table + size_t(seq) * p.max_pages;
      for (int t0 = t_begin; t0 < t_end; t0 += kDecTile) {
        if (!mbar_wait(&empty[slot], phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        int page = -1;
        bool valid = false, bad = false;
        int in_page = 0;
        if (lane < nchunks) {
          const int p0 = t0 + lane * p.chunk;
          if (p0 < len) {
            page = __ldg(&bt_row[p0 / p.page_size]);
            in_page = p0 % p.page_size;
            valid = page >= 0 && page < p.num_pages;
            bad = !valid;
          }
        }
        const uint32_t valid_mask = __ballot_sync(0xffffffffu, valid);
        const uint32_t bad_mask = __ballot_sync(0xffffffffu, bad);
        if (lane == 0) {
          if (bad_mask) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
          info[slot] = make_int2(min(kDecTile, len - t0), int(bad_mask));
          mbar_arrive_expect_tx(&full[slot], __popc(valid_mask) * chunk_bytes * 2);
        }
        __syncwarp();
        if (valid) {
          uint8_t* kdst = smem + slot * L::kStageBytes + lane * chunk_bytes;
          uint8_t* vdst = kdst + kDecTile * D * 2;
          tma_load_4d(kdst, &tm_k, &full[slot], 0, kvh, in_page, page);
          tma_load_4d(vdst, &tm_v, &full[slot], 0, kvh, in_page, page);
        }
        pending |= 1u << slot;
        pending_phase = (pending_phase & ~(1u << slot)) | (phase << slot);
        if (++slot == kDecStages) { slot = 0; phase ^= 1u; }
      }
    }
    if (!ok && lane == 0) {
      for (int s = 0; s < kDecStages; ++s)
        if (pending & (1u << s)) mbar_drain(&full[s], (pending_phase >> s) & 1u);
    }
  } else {
    // ------------------------------------------------------------ consumer warps
    int slot = 0;
    uint32_t phase = 0;
    int red_par = 0;
    int item_par = 0;
    int no_abort = 0;  // consumers stop only on their own timeout (see mbar_wait)
    bool ok = true;
    const float neg_inf = -__int_as_float(0x7f800000);
    for (long long item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      int seq, split, kvh;
      decode_item_coords(item, p.Hkv, p.max_splits, seq, split, kvh);
      int len = __ldg(&p.seq_lens[seq]);
      len = len < 0 ? 0 : min(len, capacity);
      const int t_begin = split * p.split_tokens;
      if (t_begin >= len) continue;
      const int t_end = min(t_begin + p.split_tokens, len);
      const int n_splits = (len + p.split_tokens - 1) / p.split_tokens;

      // q for the G heads of this KV head, pre-scaled into the log2 domain
      float qf[G][DL];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const __nv_bfloat16* qrow = p.q + (size_t(seq) * p.Hq + size_t(kvh) * G + h) * D;
        float x[DL];
        load_row_slice<D>(qrow, lane, x);
#pragma unroll
        for (int d = 0; d < DL; ++d) qf[h][d] = x[d] * p.scale_log2;
      }
      float m[G], l[G], acc[G][DL];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = neg_inf;
        l[h] = 0.f;
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[h][d] = 0.f;
      }
      float* my_score = score + warp * 8 * G;

      for (int t0 = t_begin; t0 < t_end; t0 += kDecTile) {
        if (!mbar_wait(&full[slot], phase, reinterpret_cast<volatile int*>(&no_abort), p.status)) {
          ok = false;
          break;
        }
        const int2 inf = info[slot];
        const int ntok = inf.x;
        const uint32_t bad = uint32_t(inf.y);
        const __nv_bfloat16* Ks = reinterpret_cast<const __nv_bfloat16*>(smem + slot * L::kStageBytes);
        const __nv_bfloat16* Vs = Ks + kDecTile * D;

        // ---- scores of this warp's 8 tokens, reduce-scattered over the lanes
#pragma unroll
        for (int bch = 0; bch < NB; ++bch) {
          float val[V];
#pragma unroll
          for (int tk = 0; tk < TBc; ++tk) {
            float kx[DL];
            load_row_slice<D>(Ks + (warp * 8 + bch * TBc + tk) * D, lane, kx);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              float s = 0.f;
#pragma unroll
              for (int d = 0; d < DL; ++d) s = fmaf(qf[h][d], kx[d], s);
              val[tk * G + h] = s;
            }
          }
          int cur = V;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) {
            if (cur > 1) {
              const int half = cur >> 1;
              const bool upper = (lane & off) != 0;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                if (i < half) {
                  const float send = upper ? val[i] : val[i + half];
                  const float keep = upper ? val[i + half] : val[i];
                  val[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
              }
              cur = half;
            } else {
              val[0] += __shfl_xor_sync(0xffffffffu, val[0], off);
            }
          }
          // lane owns value index v = lane / DUP of this batch
          if ((lane % DUP) == 0) {
            const int v = lane / DUP;
            const int tk = v / G;
            const int tok = warp * 8 + bch * TBc + tk;
            const bool vis = tok < ntok && !((bad >> (tok / p.chunk)) & 1u);
            my_score[(bch * TBc) * G + v] = vis ? val[0] : neg_inf;
          }
        }
        __syncwarp();
        // ---- per-head max over this warp's tokens, then over the warps
        if (lane < G) {
          float mx = neg_inf;
#pragma unroll
          for (int tk = 0; tk < 8; ++tk) mx = fmaxf(mx, my_score[tk * G + lane]);
          red[(red_par * kDecConsumerWarps + warp) * G + lane] = mx;
        }
        named_bar_sync(1, kDecConsumerWarps * 32);
        float rmax_l = neg_inf;
        if (lane < G) {
#pragma unroll
          for (int w = 0; w < kDecConsumerWarps; ++w)
            rmax_l = fmaxf(rmax_l, red[(red_par * kDecConsumerWarps + w) * G + lane]);
        }
        red_par ^= 1;
        float r[G];
#pragma unroll
        for (int h = 0; h < G; ++h) r[h] = __shfl_sync(0xffffffffu, rmax_l, h);

        bool skip = false;
        if constexpr (SKIP) {
          bool all_ok = true;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const bool row_ok = (r[h] == neg_inf) || (m[h] != neg_inf && (r[h] - m[h]) < p.log2_lambda);
            all_ok = all_ok && row_ok;
          }
          skip = all_ok;
          if (p.skip_mask && warp == 0 && lane == 0)
            p.skip_mask[(size_t(seq) * p.Hkv + kvh) * p.max_tiles + t0 / kDecTile] = skip ? 1 : 0;
        }
        if (!skip) {
          float mnew[G], alpha[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            mnew[h] = fmaxf(m[h], r[h]);
            alpha[h] = (m[h] == neg_inf) ? 0.f : fast_exp2(m[h] - mnew[h]);
          }
          // probabilities of the owned scores, in place
          if ((lane % DUP) == 0) {
#pragma unroll
            for (int bch = 0; bch < NB; ++bch) {
              const int v = lane / DUP;
              const int h = v % G;
              float* sp = &my_score[(bch * TBc) * G + v];
              const float s = *sp;
              float mh = mnew[0];
#pragma unroll
              for (int hh = 1; hh < G; ++hh)
                if (h == hh) mh = mnew[hh];
              *sp = (s == neg_inf || mh == neg_inf) ? 0.f : fast_exp2(s - mh);
            }
          }
          __syncwarp();
#pragma unroll
          for (int h = 0; h < G; ++h) {
            l[h] *= alpha[h];
#pragma unroll
            for (int d = 0; d < DL; ++d) acc[h][d] *= alpha[h];
            m[h] = mnew[h];
          }
          // ---- P.V over this warp's tokens
#pragma unroll
          for (int tk = 0; tk < 8; ++tk) {
            const int tok = warp * 8 + tk;
            const bool vis = tok < ntok && !((bad >> (tok / p.chunk)) & 1u);
            if (vis) {
              float vx[DL];
              load_row_slice<D>(Vs + tok * D, lane, vx);
#pragma unroll
              for (int h = 0; h < G; ++h) {
                const float pr = my_score[tk * G + h];
                l[h] += pr;
#pragma unroll
                for (int d = 0; d < DL; ++d) acc[h][d] = fmaf(pr, vx[d], acc[h][d]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == kDecStages) { slot = 0; phase ^= 1u; }
      }
      if (!ok) break;

      // ---- combine the eight warps' (l, O) for this item and write the split result
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int d = 0; d < DL; ++d) atomicAdd(&comb_o[h * D + lane * DL + d], acc[h][d]);
        if (lane == 0) atomicAdd(&comb_l[item_par * G + h], l[h]);
      }
      named_bar_sync(1, kDecConsumerWarps * 32);
      const int tid = threadIdx.x;
      for (int i = tid; i < G * D; i += kDecConsumerWarps * 32) {
        const int h = i / D, d = i % D;
        const float lsum = comb_l[item_par * G + h];
        const float val = lsum > 0.f ? comb_o[i] / lsum : 0.f;  // 0 only if every page was invalid
        comb_o[i] = 0.f;
        const int hq = kvh * G + h;
        if (n_splits == 1)
          p.o[(size_t(seq) * p.Hq + hq) * D + d] = __float2bfloat16_rn(val);
        else
          p.ws_o[((size_t(seq) * p.max_splits + split) * p.Hq + hq) * D + d] = val;
      }
      if (tid < G) {
        const float lsum = comb_l[item_par * G + tid];
        float mh = m[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh)
          if (tid == hh) mh = m[hh];
        const float lse2 = lsum > 0.f ? mh + __log2f(lsum) : -__int_as_float(0x7f800000);
        const int hq = kvh * G + tid;
        if (n_splits == 1) {
          if (p.lse) p.lse[size_t(seq) * p.Hq + hq] = lse2 * 0.69314718055994531f;
        } else {
          p.ws_lse[(size_t(seq) * p.max_splits + split) * p.Hq + hq] = lse2;
        }
        comb_l[(item_par ^ 1) * G + tid] = 0.f;
      }
      item_par ^= 1;
    }
  }
  __syncwarp();
  __syncthreads();
}

// One warp per (sequence, query head): combine the split partials.
template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const DecodeParams p) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const long long idx = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (idx >= (long long)p.num_seqs * p.Hq) return;
  const int seq = int(idx / p.Hq), hq = int(idx % p.Hq);
  const int capacity = p.max_pages * p.page_size;
  int len = __ldg(&p.seq_lens[seq]);
  len = len < 0 ? 0 : min(len, capacity);
  const int n_splits = (len + p.split_tokens - 1) / p.split_tokens;
  __nv_bfloat16* orow = p.o + (size_t(seq) * p.Hq + hq) * D;
  const float neg_inf = -__int_as_float(0x7f800000);
  if (n_splits == 1) return;  // written by the split kernel
  if (n_splits == 0) {
#pragma unroll
    for (int d = 0; d < DL; ++d) orow[lane * DL + d] = __float2bfloat16_rn(0.f);
    if (p.lse && lane == 0) p.lse[size_t(seq) * p.Hq + hq] = neg_inf;
    return;
  }
  const float* lse_base = p.ws_lse + size_t(seq) * p.max_splits * p.Hq + hq;
  float mx = neg_inf;
  for (int s = lane; s < n_splits; s += 32) mx = fmaxf(mx, lse_base[size_t(s) * p.Hq]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float acc[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) acc[d] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float w = fast_exp2(lse_base[size_t(s) * p.Hq] - mx);
    const float* orow_s = p.ws_o + ((size_t(seq) * p.max_splits + s) * p.Hq + hq) * D + lane * DL;
    wsum += w;
#pragma unroll
    for (int d = 0; d < DL; ++d) acc[d] = fmaf(w, orow_s[d], acc[d]);
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int d = 0; d < DL; ++d) orow[lane * DL + d] = __float2bfloat16_rn(acc[d] * inv);
  if (p.lse && lane == 0) p.lse[size_t(seq) * p.Hq + hq] = (mx + __log2f(wsum)) * 0.69314718055994531f;
}

}  // namespace attn
