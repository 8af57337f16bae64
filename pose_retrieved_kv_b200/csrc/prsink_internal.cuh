// Internal helpers shared by the prsink CUDA sources: host-side error text and launch count,
// the device status word, bounded mbarrier waits and thin PTX wrappers for sm_100a
// (mbarrier, TMA, tcgen05).  Nothing here is part of the C ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/prsink.h"

namespace prsink {

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
void set_error(const char* fmt, ...);
int check_launch(const char* what);          // PRSINK_OK or PRSINK_ERR_LAUNCH (+ text)
void count_launch(int n = 1);
int* status_word_ptr();                      // device address of the status word (per device)

struct Geometry {                            // derived token counts of a layout
  long long L_f, L_blk, L_ref, T;
  int n_slots;                               // 3 + R
  long long slot_start[3 + PRSINK_MAX_RING + 1];
};
int geometry(const prsink_layout* L, Geometry* g);   // validates, PRSINK_OK or ERR_ARG

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D bf16 TMA tensor map (dims d0 x d1 x d2, strides in bytes for dims 1 and 2) with a
// 64 x box1 x box2 box, 128-byte swizzle, zero fill out of bounds.  PRSINK_OK or ERR_LAUNCH.
int make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2);

// ------------------------------------------------------------------------------------------
// device side
// ------------------------------------------------------------------------------------------
constexpr int kStatusTimeout = 1;

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Shared abort state of one CTA: set by the first wait that runs out, seen by all others.
struct AbortState {
  volatile int flag;
};

// Wait until the barrier's phase with the given parity has completed.  Gives up when the
// CTA-wide abort flag is set or the deadline (globaltimer, ns) passes; in the latter case it
// records the timeout in the device status word and raises the abort flag.  Returns true when
// the phase completed.
// The first try_wait stands alone, outside the loop: in a reconstruction of the attention
// kernel's hand-offs (MMA issuer, softmax, rotation and producer warps, no arithmetic) the
// single-loop form cost ~50 cycles more per wait (2624 against 2315 cycles per key tile); the
// kernel itself runs ~1 % faster with this form.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, AbortState* ab,
                                          uint64_t deadline, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++spins & 1023u) == 0) {
      if (ab->flag) return false;
      if (globaltimer() > deadline) {
        ab->flag = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
  return true;
}

// bar.sync on named barrier `id` (1..15) for `count` threads (a multiple of 32): a barrier for
// a subset of the CTA's warps
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// bar.red.and on named barrier `id` for `count` threads: true iff `pred` holds in all of them
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r) : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count) : "memory");
  return r != 0;
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA: 3-D tiled load into shared memory, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :: "r"(dst), "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

// TMA: 3-D tiled store from shared memory (bulk-group completion).  The tile must have been
// written through the async proxy, or be followed by fence.proxy.async before this call.
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               :: "l"(tmap), "r"(src), "r"(c0), "r"(c1), "r"(c2) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store group of this thread but the newest has finished
// reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all_but_newest() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until every committed bulk store of this thread has completed (writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// ---- tcgen05 (5th-generation tensor core, tensor memory) -------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, f32 accumulate).
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrive once on an mbarrier when every tcgen05.mma issued so far by this thread completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane -> registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
         "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
         "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
         "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
         "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading / stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;                 // version (sm_100)
  d |= 2ull << 61;                 // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, f32 accumulator, M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4)                                  // D format f32
       | (1u << 7)                                  // A format bf16
       | (1u << 10)                                 // B format bf16
       | (static_cast<uint32_t>(a_mn_major) << 15)
       | (static_cast<uint32_t>(b_mn_major) << 16)
       | (static_cast<uint32_t>(N >> 3) << 17)
       | (static_cast<uint32_t>(M >> 4) << 24);
}

}  // namespace prsink

namespace prsink {
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16; A is M x 16 in 8 TMEM columns (bf16 pairs).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane <- registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
         "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
         "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// S = A B^T over K = 128 (eight K = 16 steps) with A and B K-major, 128-byte swizzled in two
// 64-column panels 16 KB apart: descriptor of step kk = base + (kk / 4) * 16 KB + (kk % 4) * 32 B,
// i.e. +1024 or +2 in the descriptor's 16-byte address units.  Step 0 overwrites D.  One asm
// block keeps the issuing thread at a few instructions per MMA.
__device__ __forceinline__ void umma_ss_k128(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, 0, 0;\n\tsetp.eq.b32 p1, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n\t"
      "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 1024;\n\tadd.s64 b, %2, 1024;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 1026;\n\tadd.s64 b, %2, 1026;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 1028;\n\tadd.s64 b, %2, 1028;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 1030;\n\tadd.s64 b, %2, 1030;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(idesc) : "memory");
}
// Same over K = 64 (four steps, one panel).
__device__ __forceinline__ void umma_ss_k64(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, 0, 0;\n\tsetp.eq.b32 p1, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n\t"
      "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t"
      "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p1;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(idesc) : "memory");
}
// O (+)= P V over 128 keys (eight K = 16 steps): P in TMEM (8 columns per step), V MN-major in
// shared memory (8 key rows of 128 B per 1 KB atom: step kk = base + kk * 2 KB, +128 units).
// The first step accumulates only if `acc` is non-zero.
__device__ __forceinline__ void umma_ts_pv128(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                              uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\tsetp.eq.b32 p1, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
      "add.s32 a, %1, 8;\n\tadd.s64 b, %2, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 16;\n\tadd.s64 b, %2, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 24;\n\tadd.s64 b, %2, 384;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 32;\n\tadd.s64 b, %2, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 40;\n\tadd.s64 b, %2, 640;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 48;\n\tadd.s64 b, %2, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t"
      "add.s32 a, %1, 56;\n\tadd.s64 b, %2, 896;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p1;\n\t}"
      :: "r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(N));
}
// Packed float32 pair arithmetic (sm_100): two lanes of fp32 per instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
}  // namespace prsink
