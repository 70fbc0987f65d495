// C ABI of the attention library: argument validation, TMA descriptor
// encoding and kernel launches. Everything is enqueued on the caller's stream;
// nothing here allocates device memory or synchronises (except
// attn_read_device_status, which is documented to).
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "decode.cuh"
#include "decode_heads.cuh"
#include "decode_blasst.cuh"
#include "decode_gate.cuh"
#include "kv_append.cuh"
#include "prefill.cuh"

using namespace attn;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

// Current device's SM count; ATTN_ERR_UNSUPPORTED unless it is compute capability 10.0.
int current_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.ready) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.sms = count;
    d.ready = true;
  }
  if (!d.supported) return ATTN_ERR_UNSUPPORTED;
  *sms = d.sms;
  return ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4-D tensor map (bf16 unless told otherwise). dims/box innermost first; strides in bytes for dims 1..3.
int encode_map(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
               const uint32_t box[4], CUtensorMapSwizzle swizzle,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return ATTN_ERR_CUDA;
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t s[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
  const CUresult r = enc(map, dtype, 4, const_cast<void*>(base), d, s, b, elem_strides,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID_ARG;
}

// 5-D bf16 tensor map with the 128-byte swizzle. dims/box innermost first; strides in bytes for dims 1..4.
int encode_map5(CUtensorMap* map, const void* base, const uint64_t dims[5], const uint64_t strides[4],
                const uint32_t box[5]) {
  auto enc = tensor_map_encoder();
  if (!enc) return ATTN_ERR_CUDA;
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  cuuint64_t d[5] = {dims[0], dims[1], dims[2], dims[3], dims[4]};
  cuuint64_t s[4] = {strides[0], strides[1], strides[2], strides[3]};
  cuuint32_t b[5] = {box[0], box[1], box[2], box[3], box[4]};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), d, s, b, elem_strides,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID_ARG;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device and kernel (one mask per kernel, keyed by the kernel itself): check that it
// was compiled with at least `min_regs` registers per thread (0: no check) and raise its
// dynamic shared-memory limit. The launch path then makes no attribute call, which keeps it
// a plain sequence of stream operations under graph capture and saves host time per launch.
template <auto kernel>
int set_smem_once(int smem, int min_regs = 0) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return ATTN_OK;
  if (min_regs > 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return ATTN_ERR_CUDA;
    if (attr.numRegs < min_regs) return ATTN_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return ATTN_OK;
}

// [B][S][H][D] bf16 tensor as a 4-D map {D, S, H, B}; box = 64 columns x `rows` rows of one head.
int encode_bshd(CUtensorMap* map, const void* base, int B, int S, int H, int D, int rows = kPfRows) {
  const uint64_t dims[4] = {uint64_t(D), uint64_t(S), uint64_t(H), uint64_t(B)};
  const uint64_t strides[3] = {uint64_t(H) * D * 2, uint64_t(D) * 2, uint64_t(S) * H * D * 2};
  const uint32_t box[4] = {64, uint32_t(rows), 1, 1};
  return encode_map(map, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

template <int D, bool CAUSAL, bool SKIP, bool PAGED = false, bool DBG = false>
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tvh,
                   const PrefillParams& p, int sms, cudaStream_t stream) {
  auto kernel = prefill_kernel<D, CAUSAL, SKIP, PAGED, DBG>;
  constexpr int smem = PrefillSmem<D>::kDynamic;
  // The kernel moves registers between warpgroups with setmaxnreg; the block's
  // launch allocation must cover the split or the increase would never return
  // (checked with the shared-memory limit, once per device).
  if (int st = set_smem_once<prefill_kernel<D, CAUSAL, SKIP, PAGED, DBG>>(
          smem, (kPfRegPoolNeeded + kPfThreads - 1) / kPfThreads))
    return st;
  const long long grid = p.num_items < sms ? p.num_items : sms;
  kernel<<<dim3(unsigned(grid)), dim3(kPfThreads), smem, stream>>>(tq, tk, tv, tvh, p);
  return launch_status();
}

template <int D, bool SKIP>
int dispatch_prefill_causal(bool causal, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tvh, const PrefillParams& p, int sms, cudaStream_t stream) {
  return causal ? launch_prefill<D, true, SKIP>(tq, tk, tv, tvh, p, sms, stream)
                : launch_prefill<D, false, SKIP>(tq, tk, tv, tvh, p, sms, stream);
}

// Pipeline settings that only the test entry point changes.
struct PrefillDebug {
  unsigned long long wait_ns = kWaitLimitNs;
  int withhold_step = -1;
};

int prefill_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int S,
                 int D, int causal, float scale, float lambda, uint8_t* skip_mask,
                 unsigned long long* skipped_tiles, int* device_status, void* stream, bool blasst,
                 const PrefillDebug& dbg = PrefillDebug()) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(skipped_tiles) & 7u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda < 1.f)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * S * Hq > (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  int sms = 0;
  if (int st = current_device(&sms)) return st;

  PrefillParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.skip_mask = skip_mask;
  p.skipped_tiles = skipped_tiles;
  p.status = device_status;
  p.wait_ns = dbg.wait_ns;
  p.withhold_step = dbg.withhold_step;
  p.B = B; p.S = S; p.Hq = Hq; p.Hkv = Hkv;
  p.n_qblocks = (S + 2 * kPfRows - 1) / (2 * kPfRows);
  p.n_qt = (S + kPfRows - 1) / kPfRows;
  p.n_kt = (S + 63) / 64;
  const long long num_items = (long long)p.n_qblocks * B * Hq;
  if (num_items > 0x7fffffffll) return ATTN_ERR_UNSUPPORTED;
  p.num_items = int(num_items);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.log2_lambda = lambda > 0.f ? std::log2(lambda) : -INFINITY;

  CUtensorMap tq, tk, tv, tvh;
  if (int st = encode_bshd(&tq, q, B, S, Hq, D)) return st;
  if (int st = encode_bshd(&tk, k, B, S, Hkv, D)) return st;
  if (int st = encode_bshd(&tv, v, B, S, Hkv, D)) return st;
  if (int st = encode_bshd(&tvh, v, B, S, Hkv, D, kPfKeys / 2)) return st;   // one 64-key half per box
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the mask and the count need the decision path
  const bool use_skip = blasst && (lambda > 0.f || skip_mask != nullptr || skipped_tiles != nullptr);
  if (dbg.withhold_step >= 0 || dbg.wait_ns != kWaitLimitNs) {   // the test entry point (dense only)
    if (D == 128)
      return causal ? launch_prefill<128, true, false, false, true>(tq, tk, tv, tvh, p, sms, s)
                    : launch_prefill<128, false, false, false, true>(tq, tk, tv, tvh, p, sms, s);
    return causal ? launch_prefill<64, true, false, false, true>(tq, tk, tv, tvh, p, sms, s)
                  : launch_prefill<64, false, false, false, true>(tq, tk, tv, tvh, p, sms, s);
  }
  if (D == 128)
    return use_skip ? dispatch_prefill_causal<128, true>(causal != 0, tq, tk, tv, tvh, p, sms, s)
                    : dispatch_prefill_causal<128, false>(causal != 0, tq, tk, tv, tvh, p, sms, s);
  return use_skip ? dispatch_prefill_causal<64, true>(causal != 0, tq, tk, tv, tvh, p, sms, s)
                  : dispatch_prefill_causal<64, false>(causal != 0, tq, tk, tv, tvh, p, sms, s);
}

// Page pool [P][page_size][Hkv][D] as a 4-D map {D, Hkv, page_size, P}; box =
// 64 columns x 16 slots of one head (a page size is a multiple of 16).
int encode_pool16(CUtensorMap* map, const void* base, int P, int page_size, int Hkv, int D) {
  const uint64_t dims[4] = {uint64_t(D), uint64_t(Hkv), uint64_t(page_size), uint64_t(P)};
  const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(Hkv) * D * 2, uint64_t(page_size) * Hkv * D * 2};
  const uint32_t box[4] = {64, 1, 16, 1};
  return encode_map(map, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool valid_prefill_page_size(int ps) { return ps == 16 || ps == 32 || ps == 64 || ps == 128 || ps == 256; }

// ------------------------------------------------------------------ decode

// decode workspace: [work-ticket counter, 256 B][partial O][partial log2-sum-exp]
constexpr size_t kWsHeader = 256;

bool valid_page_size(int ps) { return ps == 16 || ps == 32 || ps == 64 || ps == 128 || ps == 256; }

long long max_splits_of(int max_pages, int page_size, int split_tokens) {
  const long long cap = (long long)max_pages * page_size;
  return (cap + split_tokens - 1) / split_tokens;
}

// a * b into *out; false when the product does not fit a size_t
bool mul_size(size_t a, size_t b, size_t* out) { return !__builtin_mul_overflow(a, b, out); }
bool add_size(size_t a, size_t b, size_t* out) { return !__builtin_add_overflow(a, b, out); }

// Bytes of the decode workspace [header][partial O][partial log2-sum-exp] for `slots`
// (sequence, split) pairs; 0 when a size overflows. *o_bytes receives the partial-O bytes.
size_t decode_ws_bytes(size_t slots, size_t Hq, size_t D, size_t* o_bytes) {
  size_t rows = 0, ob = 0, lb = 0, total = 0;
  if (!mul_size(slots, Hq, &rows) || !mul_size(rows, D * sizeof(float), &ob) || !mul_size(rows, sizeof(float), &lb))
    return 0;
  if (!add_size(ob, 255, &total)) return 0;
  const size_t ob_aligned = total / 256 * 256;
  if (!add_size(kWsHeader, ob_aligned, &total) || !add_size(total, lb, &total)) return 0;
  if (o_bytes) *o_bytes = ob;
  return total;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// Workspace of the two-pass tile-skip decode, every part 256-byte aligned:
//   [header: two work-ticket counters][partial O [N][max_chunks][Hq][D]][partial lse [N][max_chunks][Hq]]
//   [scores [N][Hq][tok64]][tile maxima [N][Hq][max_tiles]][chunk maxima [N][Hq][max_chunks]]
// A work item covers chunk_tokens tokens: the largest of 256, 192, 128, 64 that divides split_tokens (so
// no chunk straddles a decision split), halved down to 64 while the batch gives fewer than 32768
// (sequence, query head, chunk) triples, so that a few long sequences still fill the GPU.
struct BlasstLayout {
  int chunk = 0, max_chunks = 0, max_tiles = 0, tok64 = 0, chunk2 = 0, max_chunks2 = 0;
  size_t o_off = 0, lse_off = 0, s_off = 0, tmax_off = 0, cmax_off = 0, cpre_off = 0, total = 0;
};

bool blasst_layout(int num_seqs, int Hq, int D, int max_pages, int page_size, int split_tokens, BlasstLayout* L) {
  if (num_seqs < 1 || Hq < 1 || (D != 64 && D != 128) || max_pages < 1 || !valid_page_size(page_size) ||
      split_tokens < 64 || split_tokens % 64 != 0)
    return false;
  const long long cap = (long long)max_pages * page_size;
  if (cap > (1ll << 30)) return false;
  int C = 64;
  for (int c : {256, 192, 128}) {
    if (split_tokens % c == 0) { C = c; break; }
  }
  L->chunk2 = C;   // pass 2's item
  L->max_chunks2 = int((cap + C - 1) / C);
  while (C % 128 == 0 && (long long)num_seqs * Hq * ((cap + C - 1) / C) < 32768) C /= 2;
  L->chunk = C;    // pass 1's item
  L->max_chunks = int((cap + C - 1) / C);
  L->max_tiles = int((cap + 63) / 64);
  L->tok64 = L->max_tiles * 64;
  const size_t rows = size_t(num_seqs) * size_t(Hq);
  size_t sz[6];
  if (!mul_size(rows, size_t(L->max_chunks2) * D * sizeof(float), &sz[0]) ||
      !mul_size(rows, size_t(L->max_chunks2) * sizeof(float), &sz[1]) ||
      !mul_size(rows, size_t(L->tok64) * sizeof(float), &sz[2]) ||
      !mul_size(rows, size_t(L->max_tiles) * sizeof(float), &sz[3]) ||
      !mul_size(rows, size_t(L->max_chunks) * sizeof(float), &sz[4]) ||
      !mul_size(rows, size_t(L->max_chunks) * sizeof(float), &sz[5]))
    return false;
  size_t off = kWsHeader;
  size_t* offs[6] = {&L->o_off, &L->lse_off, &L->s_off, &L->tmax_off, &L->cmax_off, &L->cpre_off};
  for (int i = 0; i < 6; ++i) {
    *offs[i] = off;
    size_t end = 0;
    if (!add_size(off, sz[i], &end) || !add_size(end, 255, &end)) return false;
    off = end / 256 * 256;
  }
  L->total = off;
  return true;
}

// One CTA per (sequence, query head); a no-op for sequences of one split.
// Launched as a programmatic dependent of the split kernel: it is scheduled
// while the split kernel's last CTAs run and waits (griddepcontrol.wait) for
// that grid to finish and its writes to be visible before it reads the partials.
// A row with more than 64 partials (long sequences at small splits) takes
// sixteen warps on each of D / 32 CTAs, one per 32 head dimensions (sixteen warps
// on one CTA when the partials are sparse); four warps on one CTA otherwise.
template <int D>
int launch_merge(const DecodeParams& p, cudaStream_t stream, bool sparse = false) {
  const long long pairs = (long long)p.num_seqs * p.Hq;
  const bool wide = p.max_splits > 64;
  constexpr int kSlices = D / 32;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(wide ? pairs * kSlices : pairs));
  cfg.blockDim = dim3((wide ? 16 : 4) * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (wide && sparse) {   // few O rows to read: one CTA per row, its sixteen warps on the log-sum-exps
    cfg.gridDim = dim3(unsigned(pairs));
    e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 16, 1, true>, p);
  } else if (wide)
    e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 16, kSlices, false>, p);
  else
    e = sparse ? cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 4, 1, true>, p)
               : cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 4, 1, false>, p);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  return launch_status();
}

template <int D, int G, bool SKIP>
int launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int sms,
                  cudaStream_t stream) {
  auto kernel = decode_split_kernel<D, G, SKIP>;
  constexpr int smem = DecodeSmem<D, G>::kDynamic;
  if (int st = set_smem_once<decode_split_kernel<D, G, SKIP>>(smem)) return st;
  const long long grid = p.num_items < sms ? p.num_items : sms;
  kernel<<<dim3(unsigned(grid)), dim3(kDecThreads), smem, stream>>>(tk, tv, p);
  if (int st = launch_status()) return st;
  return launch_merge<D>(p, stream);
}

template <int D, bool SKIP>
int dispatch_decode_g(int G, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int sms,
                      cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode<D, 1, SKIP>(tk, tv, p, sms, s);
    case 2: return launch_decode<D, 2, SKIP>(tk, tv, p, sms, s);
    case 4: return launch_decode<D, 4, SKIP>(tk, tv, p, sms, s);
    case 8: return launch_decode<D, 8, SKIP>(tk, tv, p, sms, s);
    case 16: return launch_decode<D, 16, SKIP>(tk, tv, p, sms, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <int D, int G, int HG, bool F8, int BLOCKS>
int launch_decode_heads_blocks(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                               int* ticket_counter, int sms, cudaStream_t stream) {
  using L = DecodeHeadsSmem<D, G, HG, F8, BLOCKS>;
  auto kernel = decode_heads_kernel<D, G, HG, F8, BLOCKS>;
  if (int st = set_smem_once<decode_heads_kernel<D, G, HG, F8, BLOCKS>>(L::kDynamic)) return st;
  const long long items = (long long)p.max_splits * p.num_seqs * (p.Hkv / HG);
  const long long slots = (long long)sms * L::kBlocks;
  const long long grid = items < slots ? items : slots;
  DecodeParams pk = p;
  pk.static_items = items <= slots ? 1 : 0;   // one item per CTA: no ticket counter to zero
  if (!pk.static_items && cudaMemsetAsync(ticket_counter, 0, sizeof(int), stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  kernel<<<dim3(unsigned(grid)), dim3((HG + 1) * 32), L::kDynamic, stream>>>(tk, tv, pk, ticket_counter);
  if (int st = launch_status()) return st;
  return launch_merge<D>(p, stream);
}

// A grid of at most two items per SM (few sequences, each with few splits) runs two CTAs
// per SM with three stages each; anything larger the default residency.
template <int D, int G, int HG, bool F8 = false>
int launch_decode_heads(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int* ticket_counter,
                        int sms, cudaStream_t stream) {
  constexpr bool kDeep = !F8 && G <= 4;   // the layouts whose default is three CTAs per SM
  if constexpr (kDeep) {
    const long long items = (long long)p.max_splits * p.num_seqs * (p.Hkv / HG);
    if (items <= 2ll * sms)
      return launch_decode_heads_blocks<D, G, HG, F8, 2>(tk, tv, p, ticket_counter, sms, stream);
  }
  return launch_decode_heads_blocks<D, G, HG, F8, 0>(tk, tv, p, ticket_counter, sms, stream);
}

// groups of 4 KV heads for G <= 8 (several CTAs per SM); G = 16 takes groups of hg (8 or 4)
template <int D>
int dispatch_decode_heads(int G, int hg, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          int* ctr, int sms, cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode_heads<D, 1, 4>(tk, tv, p, ctr, sms, s);
    case 2: return launch_decode_heads<D, 2, 4>(tk, tv, p, ctr, sms, s);
    case 4: return launch_decode_heads<D, 4, 4>(tk, tv, p, ctr, sms, s);
    case 8: return launch_decode_heads<D, 8, 4>(tk, tv, p, ctr, sms, s);
    case 16: return hg == 8 ? launch_decode_heads<D, 16, 8>(tk, tv, p, ctr, sms, s)
                            : launch_decode_heads<D, 16, 4>(tk, tv, p, ctr, sms, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// Two-pass tile-skip decode: pass 1 (scores and maxima); for splits of more than 16 chunks the scan of the
// running maxima at the chunk starts; pass 2 (decisions, kept V, P V); the merge of the chunk partials (reading
// only the non-empty ones when lambda > 0) -- each a programmatic dependent of the one before.
template <int D, int G, int HG, bool PER_HEAD>
int launch_blasst(const CUtensorMap& tk, const CUtensorMap& tvg, const CUtensorMap& tvh, const DecodeParams& p,
                  int* tickets, int sms, cudaStream_t stream) {
  using L1 = BlScoresSmem<D, G, HG>;
  using L2 = BlPvSmem<D, G, HG>;
  if (int st = set_smem_once<decode_scores_kernel<D, G, HG>>(L1::kDynamic)) return st;
  if (int st = set_smem_once<decode_pv_kernel<D, G, HG, PER_HEAD>>(L2::kDynamic)) return st;
  const long long items = (long long)p.max_chunks * p.num_seqs * (p.Hkv / HG);
  const long long items2 = (long long)p.max_chunks2 * p.num_seqs * (p.Hkv / HG);
  const long long slots1 = (long long)sms * L1::kBlocks, slots2 = (long long)sms * L2::kBlocks;
  decode_scores_kernel<D, G, HG><<<dim3(unsigned(items < slots1 ? items : slots1)), dim3((HG + 1) * 32),
                                   L1::kDynamic, stream>>>(tk, p, tickets);
  if (int st = launch_status()) return st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.ws_cpre) {   // long splits: running maxima at the chunk starts, between the passes
    const long long rows = (long long)p.num_seqs * p.Hq;
    cfg.gridDim = dim3(unsigned((rows + kScanWarps - 1) / kScanWarps));
    cfg.blockDim = dim3(kScanWarps * 32);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, decode_chunk_prefix_kernel, p) != cudaSuccess) return ATTN_ERR_CUDA;
    if (int st = launch_status()) return st;
  }
  cfg.gridDim = dim3(unsigned(items2 < slots2 ? items2 : slots2));
  cfg.blockDim = dim3((HG + 1) * 32);
  cfg.dynamicSmemBytes = L2::kDynamic;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_pv_kernel<D, G, HG, PER_HEAD>, tvg, tvh, p, tickets + 1) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (int st = launch_status()) return st;
  DecodeParams pm = p;          // the merge combines the pass-2 item partials
  pm.split_tokens = p.chunk2_tokens;
  pm.max_splits = p.max_chunks2;
  return launch_merge<D>(pm, stream, p.log2_lambda != -INFINITY);
}

template <int D, int HG, bool PER_HEAD>
int dispatch_blasst_g(int G, const CUtensorMap& tk, const CUtensorMap& tvg, const CUtensorMap& tvh,
                      const DecodeParams& p, int* tickets, int sms, cudaStream_t s) {
  switch (G) {
    case 1: return launch_blasst<D, 1, HG, PER_HEAD>(tk, tvg, tvh, p, tickets, sms, s);
    case 2: return launch_blasst<D, 2, HG, PER_HEAD>(tk, tvg, tvh, p, tickets, sms, s);
    case 4: return launch_blasst<D, 4, HG, PER_HEAD>(tk, tvg, tvh, p, tickets, sms, s);
    case 8: return launch_blasst<D, 8, HG, PER_HEAD>(tk, tvg, tvh, p, tickets, sms, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <int D>
int dispatch_blasst(int G, int hg, bool per_head, const CUtensorMap& tk, const CUtensorMap& tvg,
                    const CUtensorMap& tvh, const DecodeParams& p, int* tickets, int sms, cudaStream_t s) {
  if (hg == 4)
    return per_head ? dispatch_blasst_g<D, 4, true>(G, tk, tvg, tvh, p, tickets, sms, s)
                    : dispatch_blasst_g<D, 4, false>(G, tk, tvg, tvh, p, tickets, sms, s);
  return per_head ? dispatch_blasst_g<D, 1, true>(G, tk, tvg, tvh, p, tickets, sms, s)
                  : dispatch_blasst_g<D, 1, false>(G, tk, tvg, tvh, p, tickets, sms, s);
}

// Single-pass tile-skip decode over the splits, then the merge of the split partials.
template <int D, int G, int HG, bool PER_HEAD>
int launch_gate(const CUtensorMap& tk, const CUtensorMap& tvh, const DecodeParams& p, int* ticket_counter, int sms,
                cudaStream_t stream) {
  using L = GateSmem<D, G, HG>;
  if (int st = set_smem_once<decode_gate_kernel<D, G, HG, PER_HEAD>>(L::kDynamic)) return st;
  const long long items = (long long)p.max_splits * p.num_seqs * (p.Hkv / HG);
  const long long slots = (long long)sms * L::kBlocks;
  decode_gate_kernel<D, G, HG, PER_HEAD><<<dim3(unsigned(items < slots ? items : slots)), dim3((HG + 1) * 32),
                                           L::kDynamic, stream>>>(tk, tvh, p, ticket_counter);
  if (int st = launch_status()) return st;
  return launch_merge<D>(p, stream);
}

template <int D, int HG, bool PER_HEAD>
int dispatch_gate_g(int G, const CUtensorMap& tk, const CUtensorMap& tvh, const DecodeParams& p, int* tickets,
                    int sms, cudaStream_t s) {
  switch (G) {
    case 1: return launch_gate<D, 1, HG, PER_HEAD>(tk, tvh, p, tickets, sms, s);
    case 2: return launch_gate<D, 2, HG, PER_HEAD>(tk, tvh, p, tickets, sms, s);
    case 4: return launch_gate<D, 4, HG, PER_HEAD>(tk, tvh, p, tickets, sms, s);
    case 8: return launch_gate<D, 8, HG, PER_HEAD>(tk, tvh, p, tickets, sms, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <int D>
int dispatch_gate(int G, int hg, bool per_head, const CUtensorMap& tk, const CUtensorMap& tvh, const DecodeParams& p,
                  int* tickets, int sms, cudaStream_t s) {
  if (hg == 2)
    return per_head ? dispatch_gate_g<D, 2, true>(G, tk, tvh, p, tickets, sms, s)
                    : dispatch_gate_g<D, 2, false>(G, tk, tvh, p, tickets, sms, s);
  return per_head ? dispatch_gate_g<D, 1, true>(G, tk, tvh, p, tickets, sms, s)
                  : dispatch_gate_g<D, 1, false>(G, tk, tvh, p, tickets, sms, s);
}

// The tile-skip decode for Hq / Hkv <= 8 runs in one pass over the splits when the batch has
// at least this many (sequence, KV head, split) triples -- enough split items to keep every SM
// streaming -- and in two passes over chunks of the splits otherwise.
constexpr long long kGateMinKvSplits = 2048;

int skip_passes(int num_seqs, int Hq, int Hkv, long long max_splits) {
  if (Hq / Hkv > 8) return 1;
  return (long long)num_seqs * Hkv * max_splits >= kGateMinKvSplits ? 1 : 2;
}

// FP8 cache (D = 128): groups of 4 KV heads for G <= 8; G = 16 takes groups of hg (8 or 4)
int dispatch_decode_heads_fp8(int G, int hg, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                              int* ctr, int sms, cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode_heads<128, 1, 4, true>(tk, tv, p, ctr, sms, s);
    case 2: return launch_decode_heads<128, 2, 4, true>(tk, tv, p, ctr, sms, s);
    case 4: return launch_decode_heads<128, 4, 4, true>(tk, tv, p, ctr, sms, s);
    case 8: return launch_decode_heads<128, 8, 4, true>(tk, tv, p, ctr, sms, s);
    case 16: return hg == 8 ? launch_decode_heads<128, 16, 8, true>(tk, tv, p, ctr, sms, s)
                            : launch_decode_heads<128, 16, 4, true>(tk, tv, p, ctr, sms, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_DEVICE_BOUNDS: return "ATTN_ERR_DEVICE_BOUNDS";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

int attn_abi_version(void) { return 2; }

int attn_decode_skip_passes(int num_seqs, int Hq, int Hkv, int max_pages_per_seq, int page_size, int split_tokens) {
  if (num_seqs < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_pages_per_seq < 1 || !valid_page_size(page_size) ||
      split_tokens < 64 || split_tokens % 64 != 0)
    return 0;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return 0;
  return skip_passes(num_seqs, Hq, Hkv, max_splits_of(max_pages_per_seq, page_size, split_tokens));
}

int attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int S,
                 int D, int causal, float scale, void* stream) {
  return prefill_impl(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, scale, 0.f, nullptr, nullptr, nullptr, stream,
                      false);
}

int attn_prefill_blasst(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int S, int D, int causal, float scale, float lambda, uint8_t* skip_mask,
                        unsigned long long* skipped_tiles, int* device_status, void* stream) {
  return prefill_impl(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, scale, lambda, skip_mask, skipped_tiles,
                      device_status, stream, true);
}

int attn_debug_prefill_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                               int Hkv, int S, int D, int causal, float scale, unsigned long long wait_limit_ns,
                               int withhold_step, int* device_status, void* stream) {
  if (wait_limit_ns < 1000ull || wait_limit_ns > kWaitLimitNs) return ATTN_ERR_INVALID_ARG;
  PrefillDebug dbg;
  dbg.wait_ns = wait_limit_ns;
  dbg.withhold_step = withhold_step < 0 ? -1 : withhold_step;
  return prefill_impl(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, scale, 0.f, nullptr, nullptr, device_status,
                      stream, false, dbg);
}

int attn_set_library_status(int enable) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const int on = enable ? 1 : 0;
  if (cudaMemcpyToSymbol(g_library_status_on, &on, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                       const int32_t* seq_lens, void* o, float* lse, int B, int Sq, int Hq, int Hkv, int D,
                       int page_size, int max_pages_per_seq, int num_pages, float scale, int* device_status,
                       void* stream) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Sq < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!valid_prefill_page_size(page_size) || max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if ((long long)Sq > (long long)max_pages_per_seq * page_size) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Sq * Hq > (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  int sms = 0;
  if (int st = current_device(&sms)) return st;

  PrefillParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = device_status;
  p.B = B; p.S = Sq; p.Hq = Hq; p.Hkv = Hkv;
  p.n_qblocks = (Sq + 2 * kPfRows - 1) / (2 * kPfRows);
  p.n_qt = (Sq + kPfRows - 1) / kPfRows;
  p.n_kt = 0;
  const long long num_items = (long long)p.n_qblocks * B * Hq;
  if (num_items > 0x7fffffffll) return ATTN_ERR_UNSUPPORTED;
  p.num_items = int(num_items);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.log2_lambda = -INFINITY;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.k_pool = static_cast<const __nv_bfloat16*>(k_pages);
  p.v_pool = static_cast<const __nv_bfloat16*>(v_pages);
  p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.wait_ns = kWaitLimitNs;
  p.withhold_step = -1;

  CUtensorMap tq, tk, tv;
  if (int st = encode_bshd(&tq, q, B, Sq, Hq, D)) return st;
  if (int st = encode_pool16(&tk, k_pages, num_pages, page_size, Hkv, D)) return st;
  if (int st = encode_pool16(&tv, v_pages, num_pages, page_size, Hkv, D)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch_prefill<128, true, false, true>(tq, tk, tv, tv, p, sms, s)
                  : launch_prefill<64, true, false, true>(tq, tk, tv, tv, p, sms, s);
}

size_t attn_decode_workspace_bytes(int num_seqs, int Hq, int D, int max_pages_per_seq, int page_size,
                                   int split_tokens) {
  if (num_seqs < 1 || Hq < 1 || (D != 64 && D != 128) || max_pages_per_seq < 1 || !valid_page_size(page_size) ||
      split_tokens < 64 || split_tokens % 64 != 0)
    return 0;
  const long long ms = max_splits_of(max_pages_per_seq, page_size, split_tokens);
  size_t slots = 0;
  if (!mul_size(size_t(num_seqs), size_t(ms), &slots)) return 0;
  return decode_ws_bytes(slots, size_t(Hq), size_t(D), nullptr);
}

size_t attn_decode_blasst_workspace_bytes(int num_seqs, int Hq, int D, int max_pages_per_seq, int page_size,
                                          int split_tokens) {
  BlasstLayout L;
  if (!blasst_layout(num_seqs, Hq, D, max_pages_per_seq, page_size, split_tokens, &L)) return 0;
  const size_t dense = attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size, split_tokens);
  return dense > L.total ? dense : L.total;
}

static int decode_impl(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                       const int32_t* seq_lens, int num_seqs, int Hq, int Hkv, int D, int page_size,
                       int max_pages_per_seq, int num_pages, float scale, float lambda, int split_tokens, void* o,
                       float* lse, void* workspace, size_t workspace_bytes, uint8_t* skip_mask,
                       unsigned long long* skipped_tiles, int* device_status, void* stream, bool per_head) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned4(block_table) || !aligned4(seq_lens) || !aligned4(lse)) return ATTN_ERR_INVALID_ARG;
  if (num_seqs < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  // merge CTAs: one per (sequence, head), or one per 32 of its head dimensions
  if ((long long)num_seqs * Hq * (D / 32) > 0x7fffffffll) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!valid_page_size(page_size) || max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if (split_tokens < 64 || split_tokens % 64 != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda < 1.f)) return ATTN_ERR_INVALID_ARG;
  if ((long long)max_pages_per_seq * page_size > (1ll << 30)) return ATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return ATTN_ERR_UNSUPPORTED;
  if (!aligned8(skipped_tiles)) return ATTN_ERR_INVALID_ARG;
  const bool use_skip = lambda > 0.f || skip_mask != nullptr || skipped_tiles != nullptr || per_head;
  const size_t need = use_skip ? attn_decode_blasst_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size,
                                                                    split_tokens)
                               : attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size,
                                                             split_tokens);
  if (need == 0 || workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
  int sms = 0;
  if (int st = current_device(&sms)) return st;

  DecodeParams p{};
  p.skipped_tiles = skipped_tiles;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  const long long ms = max_splits_of(max_pages_per_seq, page_size, split_tokens);
  int* ticket_counter = static_cast<int*>(workspace);
  p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeader);
  size_t o_bytes = 0;
  decode_ws_bytes(size_t(num_seqs) * size_t(ms), size_t(Hq), size_t(D), &o_bytes);   // checked above
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeader + (o_bytes + 255) / 256 * 256);
  p.skip_mask = skip_mask;
  p.status = device_status;
  p.num_seqs = num_seqs; p.Hq = Hq; p.Hkv = Hkv;
  p.page_size = page_size; p.max_pages = max_pages_per_seq; p.num_pages = num_pages;
  p.split_tokens = split_tokens;
  p.max_splits = int(ms);
  p.max_tiles = int(((long long)max_pages_per_seq * page_size + 63) / 64);
  p.chunk = page_size < 64 ? page_size : 64;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.log2_lambda = lambda > 0.f ? std::log2(lambda) : -INFINITY;
  p.per_head = per_head ? 1 : 0;
  p.num_items = (long long)num_seqs * ms * Hkv;

  // page pool [P][page_size][Hkv][D] as a 5-D map {64, D/64, Hkv, page_size, P}; box = the whole head
  // dimension of one head for `chunk` tokens, written as 128-byte rows with the 128-byte swizzle
  const uint64_t dims[5] = {64, uint64_t(D / 64), uint64_t(Hkv), uint64_t(page_size), uint64_t(num_pages)};
  const uint64_t strides[4] = {128, uint64_t(D) * 2, uint64_t(Hkv) * D * 2, uint64_t(page_size) * Hkv * D * 2};
  const uint32_t box[5] = {64, uint32_t(D / 64), 1, uint32_t(p.chunk), 1};
  CUtensorMap tk, tv;
  if (int st = encode_map5(&tk, k_pages, dims, strides, box)) return st;
  if (int st = encode_map5(&tv, v_pages, dims, strides, box)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int hg = G <= 8 ? (Hkv % 4 == 0 ? 4 : 0) : (Hkv % 8 == 0 ? 8 : (Hkv == 4 ? 4 : 0));
  // {64 columns, token, 64-column half, head, page}: a head's 16 tokens land as [half][token][64]
  const uint64_t hdims[5] = {64, uint64_t(page_size), uint64_t(D / 64), uint64_t(Hkv), uint64_t(num_pages)};
  const uint64_t hstrides[4] = {uint64_t(Hkv) * D * 2, 128, uint64_t(D) * 2, uint64_t(page_size) * Hkv * D * 2};
  if (use_skip && G <= 8 && skip_passes(num_seqs, Hq, Hkv, ms) == 1) {
    // one pass over the splits, groups of 2 KV heads (of 1 when Hkv is odd); V rows per head
    const int ghg = Hkv % 2 == 0 ? 2 : 1;
    const uint32_t gbox[5] = {64, uint32_t(kDhChunk), uint32_t(D / 64), uint32_t(ghg), 1};
    const uint32_t box1[5] = {64, uint32_t(kDhChunk), uint32_t(D / 64), 1, 1};
    CUtensorMap gk, gvh;
    if (int st = encode_map5(&gk, k_pages, hdims, hstrides, gbox)) return st;
    if (int st = encode_map5(&gvh, v_pages, hdims, hstrides, box1)) return st;
    if (cudaMemsetAsync(ticket_counter, 0, sizeof(int), s) != cudaSuccess) return ATTN_ERR_CUDA;
    if (D == 128) return dispatch_gate<128>(G, ghg, per_head, gk, gvh, p, ticket_counter, sms, s);
    return dispatch_gate<64>(G, ghg, per_head, gk, gvh, p, ticket_counter, sms, s);
  }
  if (use_skip && G <= 8) {
    // two passes over groups of 4 KV heads (of 1 when Hkv is not a multiple of 4)
    const int bhg = Hkv % 4 == 0 ? 4 : 1;
    BlasstLayout BL;
    blasst_layout(num_seqs, Hq, D, max_pages_per_seq, page_size, split_tokens, &BL);   // checked above
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.ws_o = reinterpret_cast<float*>(ws + BL.o_off);
    p.ws_lse = reinterpret_cast<float*>(ws + BL.lse_off);
    p.ws_s = reinterpret_cast<float*>(ws + BL.s_off);
    p.ws_tmax = reinterpret_cast<float*>(ws + BL.tmax_off);
    p.ws_cmax = reinterpret_cast<float*>(ws + BL.cmax_off);
    // splits of more than 16 chunks: the running maximum at each chunk start is scanned between the passes
    p.ws_cpre = split_tokens / BL.chunk > 16 ? reinterpret_cast<float*>(ws + BL.cpre_off) : nullptr;
    p.chunk_tokens = BL.chunk;
    p.max_chunks = BL.max_chunks;
    p.chunk2_tokens = BL.chunk2;
    p.max_chunks2 = BL.max_chunks2;
    p.tok64 = BL.tok64;
    const uint32_t gbox[5] = {64, uint32_t(kDhChunk), uint32_t(D / 64), uint32_t(bhg), 1};
    const uint32_t box1[5] = {64, uint32_t(kDhChunk), uint32_t(D / 64), 1, 1};
    CUtensorMap bk, bvg, bvh;
    if (int st = encode_map5(&bk, k_pages, hdims, hstrides, gbox)) return st;
    if (int st = encode_map5(&bvg, v_pages, hdims, hstrides, gbox)) return st;
    if (int st = encode_map5(&bvh, v_pages, hdims, hstrides, box1)) return st;
    if (cudaMemsetAsync(ticket_counter, 0, 2 * sizeof(int), s) != cudaSuccess) return ATTN_ERR_CUDA;
    if (D == 128) return dispatch_blasst<128>(G, bhg, per_head, bk, bvg, bvh, p, ticket_counter, sms, s);
    return dispatch_blasst<64>(G, bhg, per_head, bk, bvg, bvh, p, ticket_counter, sms, s);
  }
  if (!use_skip && hg > 0) {
    // dense: one item per group of hg KV heads, 16-token stages covering all of them
    const uint32_t hbox[5] = {64, uint32_t(kDhChunk), uint32_t(D / 64), uint32_t(hg), 1};
    CUtensorMap hk, hv;
    if (int st = encode_map5(&hk, k_pages, hdims, hstrides, hbox)) return st;
    if (int st = encode_map5(&hv, v_pages, hdims, hstrides, hbox)) return st;
    if (D == 128) return dispatch_decode_heads<128>(G, hg, hk, hv, p, ticket_counter, sms, s);
    return dispatch_decode_heads<64>(G, hg, hk, hv, p, ticket_counter, sms, s);
  }
  if (D == 128)
    return use_skip ? dispatch_decode_g<128, true>(G, tk, tv, p, sms, s)
                    : dispatch_decode_g<128, false>(G, tk, tv, p, sms, s);
  return use_skip ? dispatch_decode_g<64, true>(G, tk, tv, p, sms, s)
                  : dispatch_decode_g<64, false>(G, tk, tv, p, sms, s);
}

int attn_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages, const int32_t* block_table,
                   const int32_t* start_pos, int num_seqs, int T, int Hkv, int D, int page_size,
                   int max_pages_per_seq, int num_pages, int* device_status, void* stream) {
  if (!k_new || !v_new || !k_pages || !v_pages || !block_table || !start_pos) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pages) || !aligned16(v_pages))
    return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (num_seqs < 1 || T < 1 || Hkv < 1) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!valid_page_size(page_size) || max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if ((long long)num_seqs * T > (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  int sms = 0;
  if (int st = current_device(&sms)) return st;
  KvAppendParams p{};
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_pages = static_cast<__nv_bfloat16*>(k_pages);
  p.v_pages = static_cast<__nv_bfloat16*>(v_pages);
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.status = device_status;
  p.N = num_seqs; p.T = T; p.Hkv = Hkv; p.D = D;
  p.page_size = page_size; p.max_pages = max_pages_per_seq; p.num_pages = num_pages;
  const long long rows = (long long)num_seqs * T;
  long long blocks = (rows + 7) / 8;   // eight warps per block, one token row each
  if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
  kv_append_kernel<<<dim3(unsigned(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}

int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seq_lens, int num_seqs, int Hq, int Hkv, int D, int page_size,
                      int max_pages_per_seq, int num_pages, float scale, float lambda, int split_tokens, void* o,
                      float* lse, void* workspace, size_t workspace_bytes, uint8_t* skip_mask,
                      unsigned long long* skipped_tiles, int* device_status, void* stream) {
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, num_seqs, Hq, Hkv, D, page_size,
                     max_pages_per_seq, num_pages, scale, lambda, split_tokens, o, lse, workspace, workspace_bytes,
                     skip_mask, skipped_tiles, device_status, stream, false);
}

int attn_decode_paged_blasst_heads(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int Hq,
                                   int Hkv, int D, int page_size, int max_pages_per_seq, int num_pages, float scale,
                                   float lambda, int split_tokens, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, uint8_t* skip_mask, unsigned long long* skipped_tiles,
                                   int* device_status, void* stream) {
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, num_seqs, Hq, Hkv, D, page_size,
                     max_pages_per_seq, num_pages, scale, lambda, split_tokens, o, lse, workspace, workspace_bytes,
                     skip_mask, skipped_tiles, device_status, stream, true);
}

int attn_decode_paged_fp8(const void* q, const void* k_codes, const void* v_codes, float k_scale, float v_scale,
                          const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int Hq, int Hkv, int D,
                          int page_size, int max_pages_per_seq, int num_pages, float scale, int split_tokens,
                          void* o, float* lse, void* workspace, size_t workspace_bytes, int* device_status,
                          void* stream) {
  if (!q || !k_codes || !v_codes || !block_table || !seq_lens || !o || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(o) || !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned4(block_table) || !aligned4(seq_lens) || !aligned4(lse)) return ATTN_ERR_INVALID_ARG;
  if (num_seqs < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  // merge CTAs: one per (sequence, head), or one per 32 of its head dimensions
  if ((long long)num_seqs * Hq * (D / 32) > 0x7fffffffll) return ATTN_ERR_INVALID_ARG;
  if (!valid_page_size(page_size) || max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if (split_tokens < 64 || split_tokens % 64 != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(k_scale) || !(k_scale > 0.f) || !std::isfinite(v_scale) || !(v_scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  if ((long long)max_pages_per_seq * page_size > (1ll << 30)) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return ATTN_ERR_UNSUPPORTED;
  // G <= 8: groups of 4 KV heads (several CTAs per SM); G = 16: groups of 8 (or all 4)
  const int hg = G <= 8 ? (Hkv % 4 == 0 ? 4 : 0) : (Hkv % 8 == 0 ? 8 : (Hkv == 4 ? 4 : 0));
  if (hg == 0) return ATTN_ERR_UNSUPPORTED;
  const size_t need = attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size, split_tokens);
  if (need == 0 || workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
  const float scale_log2 = scale * k_scale * 1.4426950408889634f;
  if (!std::isfinite(scale_log2) || !(scale_log2 > 0.f)) return ATTN_ERR_INVALID_ARG;
  int sms = 0;
  if (int st = current_device(&sms)) return st;

  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  const long long ms = max_splits_of(max_pages_per_seq, page_size, split_tokens);
  int* ticket_counter = static_cast<int*>(workspace);
  p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeader);
  size_t o_bytes = 0;
  decode_ws_bytes(size_t(num_seqs) * size_t(ms), size_t(Hq), size_t(D), &o_bytes);   // checked above
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeader + (o_bytes + 255) / 256 * 256);
  p.status = device_status;
  p.num_seqs = num_seqs; p.Hq = Hq; p.Hkv = Hkv;
  p.page_size = page_size; p.max_pages = max_pages_per_seq; p.num_pages = num_pages;
  p.split_tokens = split_tokens;
  p.max_splits = int(ms);
  p.max_tiles = int(((long long)max_pages_per_seq * page_size + 63) / 64);
  p.chunk = page_size < 64 ? page_size : 64;
  p.scale_log2 = scale_log2;
  p.log2_lambda = -INFINITY;
  p.v_scale = v_scale;
  p.num_items = (long long)num_seqs * ms * Hkv;

  // code pool [P][page_size][Hkv][128] as a 4-D map {128, page_size, Hkv, P}; box = 16 slots of hg
  // heads, each head's slots one 2 KB block of 128-byte rows under the 128-byte swizzle
  const uint64_t dims[4] = {uint64_t(D), uint64_t(page_size), uint64_t(Hkv), uint64_t(num_pages)};
  const uint64_t strides[3] = {uint64_t(Hkv) * D, uint64_t(D), uint64_t(page_size) * Hkv * D};
  const uint32_t box[4] = {uint32_t(D), uint32_t(kDhChunk), uint32_t(hg), 1};
  CUtensorMap hk, hv;
  if (int st = encode_map(&hk, k_codes, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return st;
  if (int st = encode_map(&hv, v_codes, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch_decode_heads_fp8(G, hg, hk, hv, p, ticket_counter, sms, s);
}

}  // extern "C"

// ------------------------------------------------------------------ decode without a workspace

// The fixed scratch of attn_decode_paged_noalloc (see the header): every device
// that loads the library holds it; each call's split partials are written
// before they are read, so it never needs clearing.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_noalloc_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return ATTN_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = ptr;
  }
  *out = g_noalloc_scratch_addr[dev];
  return ATTN_OK;
}
}  // namespace

extern "C" {

int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                              const int32_t* seq_lens, int num_seqs, int Hq, int Hkv, int D, int page_size,
                              int max_pages_per_seq, int num_pages, float scale, float lambda, int split_tokens,
                              void* o, float* lse, uint8_t* skip_mask, int* device_status, void* stream) {
  const bool skip_path = lambda > 0.f || skip_mask != nullptr;
  const size_t need = skip_path ? attn_decode_blasst_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size,
                                                                     split_tokens)
                                : attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size,
                                                              split_tokens);
  if (need == 0 || need > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (int st = noalloc_scratch(&scratch)) return st;
  return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_seqs, Hq, Hkv, D, page_size,
                           max_pages_per_seq, num_pages, scale, lambda, split_tokens, o, lse, scratch,
                           ATTN_NOALLOC_SCRATCH_BYTES, skip_mask, nullptr, device_status, stream);
}

int attn_read_device_status(int* status_out, int clear) {
  if (!status_out) return ATTN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  *status_out = v;
  if (clear) {
    const int zero = ATTN_OK;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // extern "C"
