// Writing the keys and values of new tokens into the paged KV cache.
//
// The cache keeps the K/V of past tokens so that each new token only adds its
// own ("TensorRT-LLM：大模型推理优化利器", section 4; "LLM推理优化技术综述",
// PART01), in fixed-size pages that a block table maps from logical to
// physical ("TensorRT对Grouped Query Attention的支持进展", section 动态形状与KV
// Cache管理). Token t of sequence b goes to position start_pos[b] + t: page
// block_table[b][pos / page_size], slot pos % page_size. A token's Hkv x D row
// is contiguous both in the new-token tensor and in its cache slot, so each
// copy is one coalesced row; the kernel is bound by HBM.
#pragma once

#include "common.cuh"

namespace attn {

struct KvAppendParams {
  const __nv_bfloat16* k_new;   // [N][T][Hkv][D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pages;       // [num_pages][page_size][Hkv][D]
  __nv_bfloat16* v_pages;
  const int32_t* block_table;   // [N][max_pages]
  const int32_t* start_pos;     // [N]
  int* status;                  // caller's device status or null
  int N, T, Hkv, D, page_size, max_pages, num_pages;
};

// One warp per (sequence, new token), grid-stride; 16-byte loads and stores.
// A position outside the block table or a page outside the pool is skipped
// and reported as ATTN_ERR_DEVICE_BOUNDS.
__global__ void __launch_bounds__(256) kv_append_kernel(const KvAppendParams p) {
  const int lane = threadIdx.x & 31;
  const long long first = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long stride = ((long long)gridDim.x * blockDim.x) >> 5;
  const long long rows = (long long)p.N * p.T;
  const int row_vecs = p.Hkv * p.D / 8;   // 16-byte vectors per token row
  for (long long r = first; r < rows; r += stride) {
    const int b = int(r / p.T), t = int(r % p.T);
    const int pos = __ldg(&p.start_pos[b]) + t;
    const int lp = pos >= 0 ? pos / p.page_size : -1;
    if (lp < 0 || lp >= p.max_pages) {
      if (lane == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
      continue;
    }
    const int page = __ldg(&p.block_table[size_t(b) * p.max_pages + lp]);
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) raise_status(p.status, ATTN_ERR_DEVICE_BOUNDS);
      continue;
    }
    const size_t dst = (size_t(page) * p.page_size + pos % p.page_size) * p.Hkv * p.D;
    const size_t src = size_t(r) * p.Hkv * p.D;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + src);
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + src);
    uint4* kd = reinterpret_cast<uint4*>(p.k_pages + dst);
    uint4* vd = reinterpret_cast<uint4*>(p.v_pages + dst);
    for (int i = lane; i < row_vecs; i += 32) {
      const uint4 kv = __ldg(ks + i), vv = __ldg(vs + i);
      kd[i] = kv;
      vd[i] = vv;
    }
  }
}

}  // namespace attn
