// KV cache writes of the PR-Sink step, all plain HBM-bound byte copies:
//   * prsink_kv_append: a block's raw K/V, token-major [n][H][d] as a QKV projection emits
//     them, into one slot of the head-major caches [H][T][d] (a transpose at 2*d-byte rows);
//   * the dynamic-sink fill (bank entry r -> dynamic slot of every layer) and the bank store
//     (ring slot of block b -> bank entry `action` of every layer), both predicated on a
//     decision that stays in device memory;
//   * the decayed bank write, bank entry <- (1 - alpha) entry + alpha block, element-wise in
//     float32 rounded to bf16, predicated the same way.
// Every thread moves 16-byte chunks; a 256-byte head row is one 16-lane run, so reads and
// writes are fully coalesced without staging through shared memory.
#include <cuda_bf16.h>

#include "prsink_internal.cuh"

namespace prsink {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// Which append kernel runs for head_dim 64 / 128 (the TMA form unless PRSINK_APPEND_TMA=0).
#ifndef PRSINK_APPEND_TMA
#define PRSINK_APPEND_TMA 1
#endif
static const bool g_append_tma = PRSINK_APPEND_TMA;

// k_new/v_new [n][H][C] 16-byte chunks -> cache [H][T][C] rows start..start+n.
__global__ void __launch_bounds__(kCopyThreads)
append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
              uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, uint32_t n_chunks,
              uint32_t H, uint32_t C, uint64_t T, uint64_t start) {
  const uint4* __restrict__ src = blockIdx.y ? v_new : k_new;
  uint4* __restrict__ dst = blockIdx.y ? v_cache : k_cache;
  const uint32_t HC = H * C;
  const uint32_t stride = gridDim.x * kCopyThreads * kCopyUnroll;
  for (uint32_t base = blockIdx.x * kCopyThreads * kCopyUnroll + threadIdx.x; base < n_chunks;
       base += stride) {
    uint4 v[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const uint32_t i = base + u * kCopyThreads;
      if (i < n_chunks) v[u] = __ldcs(src + i);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const uint32_t i = base + u * kCopyThreads;
      if (i < n_chunks) {
        const uint32_t tok = i / HC;
        const uint32_t rem = i - tok * HC;
        const uint32_t h = rem / C;
        const uint32_t c = rem - h * C;
        dst[(static_cast<uint64_t>(h) * T + start + tok) * C + c] = v[u];
      }
    }
  }
}

// Row-tiled form for C = 8 or 16 chunks per row (head_dim 64 or 128): block (x, h, kv) moves
// tokens [x*R*U, (x+1)*R*U) of head h, R = 256/C rows per pass, U passes with all loads issued
// before the stores.  No integer division: the chunk and row of a thread are a mask and a shift.
template <int C, int U>
__global__ void __launch_bounds__(kCopyThreads)
append_rows_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                   uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, uint32_t n,
                   uint32_t H, uint64_t T, uint64_t start) {
  constexpr int R = kCopyThreads / C;
  const uint4* __restrict__ src = blockIdx.z ? v_new : k_new;
  uint4* __restrict__ dst = blockIdx.z ? v_cache : k_cache;
  const uint32_t h = blockIdx.y;
  const uint32_t c = threadIdx.x & (C - 1);
  const uint32_t tok0 = blockIdx.x * (R * U) + threadIdx.x / C;
  uint4 v[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t tok = tok0 + u * R;
    if (tok < n) v[u] = __ldcs(src + (static_cast<uint64_t>(tok) * H + h) * C + c);
  }
  uint4* __restrict__ row = dst + (static_cast<uint64_t>(h) * T + start) * C + c;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t tok = tok0 + u * R;
    if (tok < n) row[static_cast<uint64_t>(tok) * C] = v[u];
  }
}

// TMA form of the append for head_dim 64 and 128: a unit is the (K|V, head, 128 tokens) tile,
// loaded token-major from k_new / v_new (box: 64 columns x 1 head x 128 tokens) into shared
// memory and stored into the slot's rows of the head-major cache (box: 64 columns x 128 rows x 1
// head; the slot map ends at the slot, so the ragged last tile is clipped).  One thread per CTA
// keeps the stages busy: it waits for a stage's load and stores it, then refills the stage of
// the PREVIOUS tile once that older store has read it, so a store never waits for itself and
// kAppendStages - 1 loads stay in flight.  Waits are bounded (status word on timeout).
constexpr int kAppendStages = 6;
constexpr int kAppendTileBytes = 128 * 256;        // one 128-row tile of head_dim 128

struct AppendMaps {
  CUtensorMap src[2];                              // k_new, v_new   (d, H, n)
  CUtensorMap dst[2];                              // slot of k_cache, v_cache  (d, n, H)
};

template <int D>
__global__ void __launch_bounds__(32, 1)
append_tma_kernel(const __grid_constant__ AppendMaps maps, int H, int tiles, int* status,
                  unsigned long long timeout_ns) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full[kAppendStages];
  __shared__ AbortState ab;
  if (threadIdx.x != 0) return;
  constexpr int kTile = D * 2 * 128;               // bytes of one unit
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  for (int i = 0; i < kAppendStages; ++i) mbar_init(smem_u32(&full[i]), 1);
  ab.flag = 0;
  fence_barrier_init();
  const int per_kv = H * tiles;
  const int units = 2 * per_kv;
  auto unit_of = [&](int k) { return static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x); };
  auto load = [&](int k) {
    const int u = unit_of(k);
    const int kv = u / per_kv, r = u - kv * per_kv, h = r / tiles, t = r - h * tiles;
    const int st = k % kAppendStages;
    const uint32_t bar = smem_u32(&full[st]);
    mbar_arrive_expect_tx(bar, kTile);
    for (int pp = 0; pp < D / 64; ++pp)
      tma_load_3d(sb + st * kAppendTileBytes + pp * 16384, &maps.src[kv], bar, pp * 64, h,
                  t * 128);
  };
  int n_mine = 0;
  while (unit_of(n_mine) < units) ++n_mine;
  int last_load = -1;                              // highest tile whose load went out
  for (int k = 0; k < n_mine && k < kAppendStages; ++k) {
    load(k);
    last_load = k;
  }
  const uint64_t deadline = globaltimer() + timeout_ns;
  int k = 0;
  for (; k < n_mine; ++k) {
    const int st = k % kAppendStages;
    if (!mbar_wait(smem_u32(&full[st]), (k / kAppendStages) & 1, &ab, deadline, status)) break;
    const int u = unit_of(k);
    const int kv = u / per_kv, r = u - kv * per_kv, h = r / tiles, t = r - h * tiles;
    for (int pp = 0; pp < D / 64; ++pp)
      tma_store_3d(&maps.dst[kv], sb + st * kAppendTileBytes + pp * 16384, pp * 64, t * 128, h);
    bulk_commit();
    if (k >= 1 && k - 1 + kAppendStages < n_mine) {
      bulk_wait_read_all_but_newest();             // the store of tile k-1 has read its stage
      load(k - 1 + kAppendStages);
      last_load = k - 1 + kAppendStages;
    }
  }
  if (ab.flag)                                     // loads still in flight land first
    for (int j = k; j <= last_load; ++j) {
      const uint64_t dl = globaltimer() + 100000000ull;
      while (!mbar_try_wait(smem_u32(&full[j % kAppendStages]), (j / kAppendStages) & 1))
        if (globaltimer() > dl) break;
    }
  bulk_wait_all();
}

// Segment copy: segment y (one (layer, k|v, head) run of `seg_chunks` contiguous chunks) from
// src + y-dependent offset to dst + y-dependent offset.  Runs only if *sel >= 0 and, when flag
// is given, *flag == want; *sel picks the bank entry on the bank side.
struct SegCopy {
  const uint4* src;
  uint4* dst;
  uint64_t seg_chunks;          // chunks per (layer, kv, head) run
  uint32_t H;
  // chunk offsets: offset = layer*L + kv*KV + head*HD (+ sel*SEL on the bank side)
  uint64_t src_layer, src_kv, src_head, src_sel, src_base;
  uint64_t dst_layer, dst_kv, dst_head, dst_sel, dst_base;
};

__global__ void __launch_bounds__(kCopyThreads)
seg_copy_kernel(SegCopy p, const int* __restrict__ sel, const int* __restrict__ flag, int want) {
  const int s = *sel;
  if (s < 0 || (flag && *flag != want)) return;
  const uint32_t y = blockIdx.y;               // = (layer*2 + kv)*H + head
  const uint32_t head = y % p.H;
  const uint32_t lk = y / p.H;
  const uint32_t kv = lk & 1u;
  const uint32_t layer = lk >> 1;
  const uint4* __restrict__ src = p.src + p.src_base + layer * p.src_layer + kv * p.src_kv +
                                  head * p.src_head + static_cast<uint64_t>(s) * p.src_sel;
  uint4* __restrict__ dst = p.dst + p.dst_base + layer * p.dst_layer + kv * p.dst_kv +
                            head * p.dst_head + static_cast<uint64_t>(s) * p.dst_sel;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kCopyThreads * kCopyUnroll;
  for (uint64_t base = static_cast<uint64_t>(blockIdx.x) * kCopyThreads * kCopyUnroll +
                       threadIdx.x;
       base < p.seg_chunks; base += stride) {
    uint4 v[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const uint64_t i = base + u * kCopyThreads;
      if (i < p.seg_chunks) v[u] = __ldcs(src + i);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const uint64_t i = base + u * kCopyThreads;
      if (i < p.seg_chunks) dst[i] = v[u];
    }
  }
}

// w_old * x + w_new * z for the 8 bf16 of a chunk: each product and the sum rounded to
// float32 (no fused multiply-add), the result rounded to bf16 (nearest even).
__device__ __forceinline__ uint32_t blend_pair(uint32_t x, uint32_t z, float w_old, float w_new) {
  const float lo = __fadd_rn(__fmul_rn(w_old, __uint_as_float(x << 16)),
                             __fmul_rn(w_new, __uint_as_float(z << 16)));
  const float hi = __fadd_rn(__fmul_rn(w_old, __uint_as_float(x & 0xFFFF0000u)),
                             __fmul_rn(w_new, __uint_as_float(z & 0xFFFF0000u)));
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Decayed bank write: dst (bank entry, read and written) <- w_old * dst + w_new * src (ring
// slot), same segments and predicate as seg_copy_kernel.
__global__ void __launch_bounds__(kCopyThreads)
seg_blend_kernel(SegCopy p, const int* __restrict__ sel, const int* __restrict__ flag, int want,
                 float w_old, float w_new) {
  const int s = *sel;
  if (s < 0 || (flag && *flag != want)) return;
  const uint32_t y = blockIdx.y;
  const uint32_t head = y % p.H;
  const uint32_t lk = y / p.H;
  const uint32_t kv = lk & 1u;
  const uint32_t layer = lk >> 1;
  const uint4* __restrict__ src = p.src + p.src_base + layer * p.src_layer + kv * p.src_kv +
                                  head * p.src_head + static_cast<uint64_t>(s) * p.src_sel;
  uint4* __restrict__ dst = p.dst + p.dst_base + layer * p.dst_layer + kv * p.dst_kv +
                            head * p.dst_head + static_cast<uint64_t>(s) * p.dst_sel;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kCopyThreads;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * kCopyThreads + threadIdx.x;
       i < p.seg_chunks; i += stride) {
    const uint4 z = __ldcs(src + i);
    uint4 x = dst[i];
    x.x = blend_pair(x.x, z.x, w_old, w_new);
    x.y = blend_pair(x.y, z.y, w_old, w_new);
    x.z = blend_pair(x.z, z.z, w_old, w_new);
    x.w = blend_pair(x.w, z.w, w_old, w_new);
    dst[i] = x;
  }
}

static int grid_for(uint64_t chunks) {
  uint64_t g = (chunks + kCopyThreads * kCopyUnroll - 1) / (kCopyThreads * kCopyUnroll);
  if (g < 1) g = 1;
  if (g > 148ull * 16) g = 148ull * 16;
  return static_cast<int>(g);
}

// Launch the predicated copy between bank entry *sel and cache slot `slot` of every layer.
// to_cache = true: bank -> cache (dynamic-sink fill); false: cache -> bank (bank store, or the
// decayed write when blend_alpha >= 0).  Runs iff *sel >= 0 and (flag null or *flag == want).
int launch_bank_cache_copy(const prsink_layout* L, const Geometry& g, int M, int n_layers,
                           const void* bank_kv, const void* cache_kv, bool to_cache, int slot,
                           const int* sel, const int* flag, int want, cudaStream_t st,
                           float blend_alpha) {
  const uint64_t C = static_cast<uint64_t>(L->head_dim) * 2 / 16;   // chunks per row
  const uint64_t H = L->n_heads;
  // cache_kv [layers][2][H][T][d]; bank_kv [layers][M][2][H][L_blk][d]
  const uint64_t cache_head = static_cast<uint64_t>(g.T) * C;
  const uint64_t cache_kv_s = H * cache_head;
  const uint64_t cache_layer = 2 * cache_kv_s;
  const uint64_t bank_head = static_cast<uint64_t>(g.L_blk) * C;
  const uint64_t bank_kv_s = H * bank_head;
  const uint64_t bank_sel = 2 * bank_kv_s;
  const uint64_t bank_layer = static_cast<uint64_t>(M) * bank_sel;
  const uint64_t slot_off = static_cast<uint64_t>(g.slot_start[slot]) * C;
  SegCopy p{};
  p.seg_chunks = bank_head;
  p.H = static_cast<uint32_t>(H);
  if (to_cache) {
    p.src = static_cast<const uint4*>(bank_kv);
    p.dst = static_cast<uint4*>(const_cast<void*>(cache_kv));
    p.src_layer = bank_layer; p.src_kv = bank_kv_s; p.src_head = bank_head; p.src_sel = bank_sel;
    p.src_base = 0;
    p.dst_layer = cache_layer; p.dst_kv = cache_kv_s; p.dst_head = cache_head; p.dst_sel = 0;
    p.dst_base = slot_off;
  } else {
    p.src = static_cast<const uint4*>(cache_kv);
    p.dst = static_cast<uint4*>(const_cast<void*>(bank_kv));
    p.src_layer = cache_layer; p.src_kv = cache_kv_s; p.src_head = cache_head; p.src_sel = 0;
    p.src_base = slot_off;
    p.dst_layer = bank_layer; p.dst_kv = bank_kv_s; p.dst_head = bank_head; p.dst_sel = bank_sel;
    p.dst_base = 0;
  }
  const uint64_t segs = static_cast<uint64_t>(n_layers) * 2 * H;
  if (segs > 65535) {
    set_error("too many (layer, k/v, head) segments: %llu", (unsigned long long)segs);
    return PRSINK_ERR_ARG;
  }
  // about 32 CTAs per SM over all segments (four waves of eight resident 256-thread CTAs), so
  // that the last wave is a small share of the copy: with one CTA per segment, 640 segments
  // (8 layers) sat unevenly on 148 SMs (4 or 5 each) and reached 0.73 of the copy peak
  uint64_t gx = (148ull * 32 + segs - 1) / segs;
  const uint64_t gmax = (bank_head + kCopyThreads * kCopyUnroll - 1) / (kCopyThreads * kCopyUnroll);
  if (gx > gmax) gx = gmax;
  if (gx < 1) gx = 1;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(segs));
  if (blend_alpha >= 0.f) {
    const float w_new = blend_alpha;
    const float w_old = 1.0f - w_new;          // float32 subtraction, as the weights are defined
    seg_blend_kernel<<<grid, kCopyThreads, 0, st>>>(p, sel, flag, want, w_old, w_new);
  } else {
    seg_copy_kernel<<<grid, kCopyThreads, 0, st>>>(p, sel, flag, want);
  }
  count_launch();
  return check_launch("bank/cache copy");
}

}  // namespace prsink

using namespace prsink;

extern "C" int prsink_kv_append(const prsink_layout* layout, const void* k_new,
                                const void* v_new, void* k_cache, void* v_cache, int dest_slot,
                                void* stream) {
  Geometry g;
  int rc = geometry(layout, &g);
  if (rc) return rc;
  if (!k_new || !v_new || !k_cache || !v_cache) {
    set_error("prsink_kv_append: null pointer");
    return PRSINK_ERR_ARG;
  }
  if (dest_slot < 0 || dest_slot >= g.n_slots) {
    set_error("prsink_kv_append: dest_slot %d out of range [0, %d)", dest_slot, g.n_slots);
    return PRSINK_ERR_ARG;
  }
  if ((layout->head_dim * 2) % 16) {
    set_error("prsink_kv_append: head_dim*2 must be a multiple of 16 bytes");
    return PRSINK_ERR_UNSUPPORTED;
  }
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) {
    set_error("prsink_kv_append: pointers must be 16-byte aligned");
    return PRSINK_ERR_ALIGN;
  }
  const uint64_t n = g.slot_start[dest_slot + 1] - g.slot_start[dest_slot];
  const uint32_t C = layout->head_dim * 2 / 16;
  const uint64_t chunks = n * layout->n_heads * C;
  if (chunks == 0) return PRSINK_OK;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* kn = static_cast<const uint4*>(k_new);
  const auto* vn = static_cast<const uint4*>(v_new);
  auto* kc = static_cast<uint4*>(k_cache);
  auto* vc = static_cast<uint4*>(v_cache);
  const uint64_t start = static_cast<uint64_t>(g.slot_start[dest_slot]);
  constexpr int kU = 4;
  if (g_append_tma && (C == 16 || C == 8)) {
    AppendMaps maps;
    const uint64_t H = layout->n_heads, D = layout->head_dim;
    const uint64_t off = 2ull * D * start;
    int rc2 = make_map(&maps.src[0], k_new, D, H, n, 2 * D, 2 * D * H, 1, 128);
    if (!rc2) rc2 = make_map(&maps.src[1], v_new, D, H, n, 2 * D, 2 * D * H, 1, 128);
    if (!rc2) rc2 = make_map(&maps.dst[0], reinterpret_cast<char*>(k_cache) + off, D, n, H,
                             2 * D, 2 * D * g.T, 128, 1);
    if (!rc2) rc2 = make_map(&maps.dst[1], reinterpret_cast<char*>(v_cache) + off, D, n, H,
                             2 * D, 2 * D * g.T, 128, 1);
    if (rc2) return rc2;
    int* sw = status_word_ptr();
    if (!sw) return PRSINK_ERR_LAUNCH;
    const int tiles = static_cast<int>((n + 127) / 128);
    const int units = 2 * layout->n_heads * tiles;
    int n_sm = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int grid = units < n_sm ? units : n_sm;
    const int smem = kAppendStages * kAppendTileBytes + 1024;
    // the attribute belongs to each instantiation: one record per head_dim and device
    static int allowed[2][64] = {{0}};
    int& ok = allowed[C == 16 ? 1 : 0][dev >= 0 && dev < 64 ? dev : 0];
    if (ok < smem) {
      cudaError_t e = C == 16
          ? cudaFuncSetAttribute(append_tma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
          : cudaFuncSetAttribute(append_tma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return check_launch("prsink_kv_append: shared memory attribute");
      ok = smem;
    }
    if (C == 16)
      append_tma_kernel<128><<<grid, 32, smem, st>>>(maps, layout->n_heads, tiles, sw,
                                                    2000000000ull);
    else
      append_tma_kernel<64><<<grid, 32, smem, st>>>(maps, layout->n_heads, tiles, sw,
                                                   2000000000ull);
  } else if (C == 16 || C == 8) {
    const uint32_t rows_per_block = (kCopyThreads / C) * kU;
    dim3 grid(static_cast<unsigned>((n + rows_per_block - 1) / rows_per_block),
              static_cast<unsigned>(layout->n_heads), 2);
    if (C == 16)
      append_rows_kernel<16, kU><<<grid, kCopyThreads, 0, st>>>(
          kn, vn, kc, vc, static_cast<uint32_t>(n), layout->n_heads, g.T, start);
    else
      append_rows_kernel<8, kU><<<grid, kCopyThreads, 0, st>>>(
          kn, vn, kc, vc, static_cast<uint32_t>(n), layout->n_heads, g.T, start);
  } else {
    dim3 grid(grid_for(chunks), 2);
    append_kernel<<<grid, kCopyThreads, 0, st>>>(kn, vn, kc, vc, static_cast<uint32_t>(chunks),
                                                 layout->n_heads, C, static_cast<uint64_t>(g.T),
                                                 start);
  }
  count_launch();
  return check_launch("prsink_kv_append");
}
