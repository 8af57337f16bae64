// Host-side plumbing of the prsink C ABI: error text, launch counter, the device status word
// that bounded waits report into, layout validation, status synchronisation and the
// bounded-wait self-test kernel.
#include <cuda.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "prsink_internal.cuh"

namespace prsink {

namespace {
thread_local char g_err[512] = {0};
std::atomic<long long> g_launches{0};

// One status word per device (a __device__ variable is instantiated on every device that
// loads the module).  Its device address is looked up once per device.
__device__ int g_status_word;
constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;
}  // namespace

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return PRSINK_ERR_LAUNCH;
  }
  return PRSINK_OK;
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int* status_word_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      set_error("cudaGetSymbolAddress(status word) failed on device %d", dev);
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 tensor map with a 64 x box1 x box2 box and 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is not available from the driver");
    return PRSINK_ERR_LAUNCH;
  }
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {64, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return PRSINK_ERR_LAUNCH;
  }
  return PRSINK_OK;
}

int geometry(const prsink_layout* L, Geometry* g) {
  if (!L) { set_error("layout is NULL"); return PRSINK_ERR_ARG; }
  if (L->n_heads < 1 || L->head_dim < 2 || (L->head_dim & 1) || L->grid_h < 1 ||
      L->grid_w < 1 || L->frames_per_block < 1 || L->ref_frames < 0 || L->ring_slots < 1 ||
      L->ring_slots > PRSINK_MAX_RING || L->block_index < 0 || !(L->rope_base > 0.f)) {
    set_error("invalid layout (heads %d, head_dim %d, grid %dx%d, frames %d, ref %d, ring %d, "
              "block %lld)", L->n_heads, L->head_dim, L->grid_h, L->grid_w,
              L->frames_per_block, L->ref_frames, L->ring_slots, L->block_index);
    return PRSINK_ERR_ARG;
  }
  if (L->rope_mode == 3) {
    const int* s = L->rope_split;
    if (s[0] < 0 || s[1] < 0 || s[2] < 0 || (s[0] | s[1] | s[2]) & 1 ||
        s[0] + s[1] + s[2] != L->head_dim) {
      set_error("rope_split (%d,%d,%d) must be even and sum to head_dim %d", s[0], s[1], s[2],
                L->head_dim);
      return PRSINK_ERR_ARG;
    }
  } else if (L->rope_mode != 1) {
    set_error("rope_mode must be 1 or 3 (got %d)", L->rope_mode);
    return PRSINK_ERR_ARG;
  }
  g->L_f = static_cast<long long>(L->grid_h) * L->grid_w;
  g->L_blk = g->L_f * L->frames_per_block;
  g->L_ref = g->L_f * L->ref_frames;
  g->n_slots = 3 + L->ring_slots;
  g->slot_start[0] = 0;
  g->slot_start[1] = g->L_ref;
  for (int s = 2; s <= g->n_slots; ++s) g->slot_start[s] = g->slot_start[s - 1] + g->L_blk;
  g->T = g->slot_start[g->n_slots];
  if (g->T > (1ll << 30) || g->L_blk * L->n_heads > (1ll << 30)) {
    set_error("layout too large (T = %lld)", g->T);
    return PRSINK_ERR_ARG;
  }
  return PRSINK_OK;
}

// A block that waits on a barrier nothing signals, until the deadline passes.
__global__ void wait_timeout_kernel(uint64_t timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ AbortState ab;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    ab.flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const uint64_t deadline = globaltimer() + timeout_ns;
  mbar_wait(b, 0, &ab, deadline, status);   // phase 0 never completes
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(b);     // complete the phase before the CTA exits
}

}  // namespace prsink

using namespace prsink;

extern "C" {

int prsink_version(void) { return 2; }

const char* prsink_last_error(void) { return g_err; }

long long prsink_launch_count(void) { return g_launches.load(); }

int prsink_layout_tokens(const prsink_layout* layout, long long* L_f, long long* L_blk,
                         long long* L_ref, long long* T) {
  Geometry g;
  int rc = geometry(layout, &g);
  if (rc) return rc;
  if (L_f) *L_f = g.L_f;
  if (L_blk) *L_blk = g.L_blk;
  if (L_ref) *L_ref = g.L_ref;
  if (T) *T = g.T;
  return PRSINK_OK;
}

int prsink_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* sw = status_word_ptr();
  if (!sw) return PRSINK_ERR_LAUNCH;
  int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, sw, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    set_error("prsink_sync_status: %s", cudaGetErrorString(e));
    return PRSINK_ERR_LAUNCH;
  }
  if (host) {
    e = cudaMemsetAsync(sw, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
      set_error("prsink_sync_status: %s", cudaGetErrorString(e));
      return PRSINK_ERR_LAUNCH;
    }
    if (host & kStatusTimeout) {
      set_error("a bounded device wait ran out");
      return PRSINK_ERR_TIMEOUT;
    }
  }
  return PRSINK_OK;
}

int prsink_debug_wait_timeout(long long timeout_ns, void* stream) {
  if (timeout_ns < 1000) timeout_ns = 1000;
  if (timeout_ns > 5000000000ll) timeout_ns = 5000000000ll;
  int* sw = status_word_ptr();
  if (!sw) return PRSINK_ERR_LAUNCH;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_ns), sw);
  count_launch();
  return check_launch("prsink_debug_wait_timeout");
}

}  // extern "C"
