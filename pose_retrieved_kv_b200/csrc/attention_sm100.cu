// PR-Sink attention for sm_100a: TMA-staged K/V tiles from the slot-indexed cache, RoPE of the
// raw keys fused between the TMA landing and the tensor-core read ("RoPE follow"), tcgen05 MMAs
// with S, P and O in tensor memory, fp32 online softmax, no materialised score matrix.
//
// One CTA computes 256 queries (two 128-row tiles Q0, Q1) of one head, ping-ponging the two
// tiles so that the tensor core works on one tile while the other tile's softmax runs.
// Warp roles (512 threads; setmaxnreg gives the softmax warps 184 registers, the rotation
// warps 64 and the producer / MMA warps 80):
//   warps 0-3   softmax of Q0, warps 4-7 softmax of Q1: thread t owns query row t (TMEM lane
//               t); it first rotates its own row of Q in shared memory, then reads S from
//               TMEM, keeps the running max and sum, writes P as bf16 back into the S columns
//               (the A operand of the P.V MMA), rescales O in TMEM when the max grew by more
//               than 2^8, and finally normalises and stores O;
//   warps 8-11  rotation: rotate every K tile in place at the keys' current logical positions
//               (interleaved RoFormer pairs, per-axis cos/sin tables in shared memory); zero
//               the K and V rows of empty slots in boundary tiles;
//   warp  12    TMA producer: K and V tiles, each through its own 2-stage ring (Q is sent by
//               warp 1 as soon as the barriers exist);
//   warp  13    MMA issuer: per key tile j, P0(j-1).V, S0(j) = Q0 K^T, P1(j-1).V, S1(j).
// Key tiles run over the physical rows of the cache: softmax attention does not depend on the
// order of the keys, only on their positions, so each key is rotated at the position of its
// logical slot and no gather is needed.  Tiles inside empty slots are skipped.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>
#include <initializer_list>
#include <mutex>

#include "prsink_internal.cuh"

namespace prsink {
namespace attn {

constexpr int BM = 128;                 // rows of one query tile (= TMEM lanes)
constexpr int NQ = 2;                   // query tiles per CTA
constexpr int BN = 128;                 // keys per tile
constexpr int kThreads = 512;
constexpr int kRotWarp0 = 8;
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kMaxSlots = 3 + PRSINK_MAX_RING;
constexpr uint32_t kTmemCols = 512;
constexpr int kTableMaxBytes = 28 * 1024;
constexpr int kMaxTiles = 1024;             // key tiles per call (T <= 131072)
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O when the max grows > 2^8
constexpr int kMaxSplit = 8;                // split CTAs per unit (key-range shares)

struct Params {
  int H, L_blk, T, L_f, grid_h, grid_w;
  int n_slots;
  int slot_start[kMaxSlots + 1];
  int slot_frame[kMaxSlots];
  unsigned valid_mask;
  int q_frame;                          // logical frame of the current block's first frame
  int rope_mode;                        // 1 or 3
  int rd[3];                            // rotated pairs per axis (1-D: D/2, 0, 0)
  int n_frames;                         // frames of the logical layout
  int tab_h_off, tab_w_off, tab_entries;  // float2 offsets of the tables
  int step_y, step_x;                   // a step of BN tokens within a frame: rows, columns
  double log2_base;
  float scale_log2;                     // log2(e) / sqrt(d)
  __nv_bfloat16* out;
  float* lse;
  const long long* dyn_src;
  int* status;
  unsigned long long timeout_ns;
  // fused form (the current block read from k_new / v_new and stored into its ring slot)
  int cur_slot;                         // ring slot of the current block (slot id), or -1
  int n_cur_tiles;                      // key tiles of the current block
  // rotation pass (prsink_rotate_sinks): slots whose rows are rotated into k_rot
  unsigned rot_mask;
  const int* rot_dyn_flag;              // dynamic slot rotated only if *flag != 0 (nullable)
  int debug_stall;                      // self-test: withhold the first S commit of query tile 0
  // work decomposition (1-D grid): units = (head, pair of query tiles), nqb per head, head-major;
  // units >= split_base run as n_split CTAs, each over an equal share of the live key tiles,
  // writing unnormalised partial results that the last of them combines
  int nqb, split_base, n_split;
  float* part_o;                        // [split units][n_split][NQ * BM][D] float32
  float2* part_ml;                      // [split units][n_split][NQ * BM] (max in log2 units, sum)
  int* part_cnt;                        // [split units] arrival counters (zero at launch)
};

// Entries of the per-CTA tile list: a key tile index and what the roles do with it.
constexpr uint16_t kTileIdx = 0x03FF;   // tile index (sink tiles: rows idx*BN..; current: tokens)
constexpr uint16_t kTileVfix = 1u << 12;   // the rotation warps touch V before the P.V MMA
constexpr uint16_t kTileStore = 1u << 13;  // this CTA stores the raw tile into the ring slot
constexpr uint16_t kTileNew = 1u << 14;    // current-block tile (from k_new / v_new)
constexpr uint16_t kTileMask = 1u << 15;   // some columns are masked (boundary or ragged tile)

enum Bar {
  B_QFULL = 0, B_QREADY = 1,
  B_KFULL = 2, B_KREADY = 4, B_KEMPTY = 6,
  B_VFULL = 8, B_VFIX = 10, B_VEMPTY = 12,
  B_SFULL = 14, B_PFULL = 16, B_ODONE = 18,
  B_FINAL = 20, B_KSTORED = 21, B_COUNT = 23      // B_KSTORED: one per K stage
};

template <int D>
struct Layout {
  static constexpr int kPanelBytes = 128 * 128;          // 128 rows x 128 B (64 bf16)
  static constexpr int kTileBytes = (D / 64) * kPanelBytes;
  static constexpr int kQ = 0;                           // NQ query tiles
  static constexpr int kK = kQ + NQ * kTileBytes;        // 2 stages
  static constexpr int kV = kK + 2 * kTileBytes;         // 2 stages
  static constexpr int kTab = kV + 2 * kTileBytes;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
  __host__ __device__ static constexpr uint32_t col_s(int qt) { return qt * 128; }        // S, then P (bf16 pairs)
  __host__ __device__ static constexpr uint32_t col_o(int qt) { return 256 + qt * D; }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Softmax exponentials on the FMA pipe for a share of the score columns (column pair i, 0..15,
// of every 32-column chunk uses the polynomial when bit i of kPolyPairs is set).  Off: measured
// on a B200 at 480x480, 1/8, 3/16, 1/4 and 1/2 of the exponentials this way were 2-48 % slower,
// because the one softmax warp per scheduler of a query tile is bound by its own issue and
// latency, not by the special-function unit.
#ifndef PRSINK_POLY_PAIRS
#define PRSINK_POLY_PAIRS 0
#endif
constexpr uint32_t kPolyPairs = PRSINK_POLY_PAIRS;
// Row max with the three-input max.f32 of sm_100 (64 instead of 120 max instructions per row
// and tile).  Off: measured no faster (fused kernel 2.7 % slower) on a B200.
#ifndef PRSINK_MAX3
#define PRSINK_MAX3 0
#endif
constexpr bool kMax3 = PRSINK_MAX3;

// 2^x for a pair, by Cody-Waite range reduction (x = n + f, n the nearest integer, taken with the
// 1.5 * 2^23 rounding constant, f in [-1/2, 1/2]) and a degree-3 polynomial minimising the
// relative error of 2^f on [-1/2, 1/2] (Remez exchange; pose_retrieved_kv_b200/exp2_poly.py
// derives the coefficients; relative error below 1.5e-4 in float32, far under the bf16
// rounding of P that follows).  2^n is added to the exponent field of p(f); x is clamped below
// at -125 so that field stays positive (2^-125 instead of ~0 is negligible next to the row sum).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;                // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(kMagic, kMagic));
  const float2 r = fadd2(t, make_float2(-kMagic, -kMagic));      // round(x), exact
  const float2 f = ffma2(r, make_float2(-1.0f, -1.0f), x);       // x - round(x), exact
  float2 q = ffma2(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                   make_float2(0.2426111251115799f, 0.2426111251115799f));
  q = ffma2(q, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
  q = ffma2(q, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  // exponent: the low bits of t hold n; (bits(t) << 23) mod 2^32 = n << 23
  return make_float2(__uint_as_float(__float_as_uint(q.x) + __float_as_uint(t.x) * 8388608u),
                     __uint_as_float(__float_as_uint(q.y) + __float_as_uint(t.y) * 8388608u));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Slot bounds held in registers for the tile-list compaction: every bound is read once with a
// constant index (loops over the slots unrolled to the compile-time maximum), so a warp tests 32
// tiles with no divergent parameter reads.
struct SlotBounds {
  int start[kMaxSlots + 1];
  __device__ __forceinline__ explicit SlotBounds(const Params& p) {
#pragma unroll
    for (int s = 0; s <= kMaxSlots; ++s) start[s] = p.slot_start[s];
  }
  // bit 0: tile n holds a key of a slot in vm; bit 1: it also holds rows of a slot not in vm or
  // rows past the cache end (the tile needs masking)
  __device__ __forceinline__ int flags(int n, unsigned vm, const Params& p) const {
    const int lo = n * BN, hi = lo + BN, hil = min(hi, p.T);
    bool live = false, full = hi <= p.T;
#pragma unroll
    for (int s = 0; s < kMaxSlots; ++s) {
      if (s < p.n_slots) {
        if ((vm >> s) & 1u) live |= start[s] < hil && start[s + 1] > lo;
        else full &= !(start[s] < hi && start[s + 1] > lo);
      }
    }
    return (live ? 1 : 0) | (full ? 0 : 2);
  }
};

__device__ __forceinline__ int slot_of(int row, const Params& p) {
  int s = 0;
  while (s + 1 < p.n_slots && row >= p.slot_start[s + 1]) ++s;
  return s;
}

// Bounded wait that ignores the abort flag (used while draining after an abort).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t ns) {
  const uint64_t dl = globaltimer() + ns;
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() > dl) break;
}

// Rotation of two adjacent pairs of one axis at once in the two lanes of the packed fp32 FMA:
// words a, b hold (x0, x1) of pairs P and P+1 as bf16 pairs; cs = (cos_P, cos_P+1, sin_P,
// sin_P+1), ns = (-sin_P, -sin_P+1).  y0 = x0 cos - x1 sin, y1 = x0 sin + x1 cos.
__device__ __forceinline__ void rot_pair2(uint32_t& a, uint32_t& b, float4 cs, float2 ns) {
  const float2 x0 = make_float2(__uint_as_float(a << 16), __uint_as_float(b << 16));
  const float2 x1 = make_float2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u));
  const float2 c = make_float2(cs.x, cs.y);
  const float2 y0 = ffma2(x1, ns, fmul2(x0, c));
  const float2 y1 = ffma2(x1, c, fmul2(x0, make_float2(cs.z, cs.w)));
  a = pack_bf16(y0.x, y1.x);
  b = pack_bf16(y0.y, y1.y);
}

__device__ __forceinline__ void rot_pair1(uint32_t& a, float c, float sn) {
  const float x0 = __uint_as_float(a << 16), x1 = __uint_as_float(a & 0xFFFF0000u);
  a = pack_bf16(x0 * c - x1 * sn, x0 * sn + x1 * c);
}

// Grouped tables of the compile-time split (3-D RoPE, d = 128): for every axis and position,
// records of two consecutive pairs: float4 (cos, cos', sin, sin') and float2 (-sin, -sin').
template <int RT, int RH>
struct Groups {
  static constexpr int RW = 64 - RT - RH;
  static constexpr int GT = (RT + 1) / 2, GH = (RH + 1) / 2, GW = (RW + 1) / 2;
};

__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts_u4(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
               :: "r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
// Loads of the RoPE tables, which do not change after the prologue: free to be scheduled.
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
  float4 v;
  asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds_f2(uint32_t a) {
  float2 v;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}

// Rotate one row (128 bf16, two 128-byte swizzled panels at shared address `tile`) at
// (frame, y, x) with the grouped tables (shared addresses `cs`, `ns`).  Pair P lives in 32-bit
// word P of the row.  Groups of two pairs always start at an even word: t pairs (0,1)..(20,21);
// h pairs (22,23)..(40,41) then 42 alone; w pair 43 alone then (44,45)..(62,63).  So no group
// crosses a 16-byte chunk and the row is processed chunk by chunk (few live registers).
template <int RT, int RH>
__device__ __forceinline__ void rotate_row_grouped(uint32_t tile, int r, int frame, int y, int x,
                                                   bool zero, uint32_t cs, uint32_t ns,
                                                   const Params& p) {
  static_assert(RT == 22 && RH == 21, "the grouping is written for the 44/42/42 split");
  using G = Groups<RT, RH>;
  const int offH = p.n_frames * G::GT, offW = offH + p.grid_h * G::GH;
  const uint32_t csT = cs + frame * G::GT * 16, nsT = ns + frame * G::GT * 8;
  const uint32_t csH = cs + (offH + y * G::GH) * 16, nsH = ns + (offH + y * G::GH) * 8;
  const uint32_t csW = cs + (offW + x * G::GW) * 16, nsW = ns + (offW + x * G::GW) * 8;
  const uint32_t row = tile + r * 128;
  const uint32_t sw = (r & 7) << 4;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t addr = row + (c >> 3) * 16384 + (((c & 7) << 4) ^ sw);
    if (zero) {
      sts_u4(addr, make_uint4(0, 0, 0, 0));
      continue;
    }
    const uint4 v = lds_u4(addr);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      const int P = 4 * c + i;                         // even word: a group or singles
      if (P < RT) {
        rot_pair2(w[i], w[i + 1], lds_f4(csT + (P / 2) * 16), lds_f2(nsT + (P / 2) * 8));
      } else if (P + 1 < RT + RH) {
        const int j = P - RT;
        rot_pair2(w[i], w[i + 1], lds_f4(csH + (j / 2) * 16), lds_f2(nsH + (j / 2) * 8));
      } else if (P < RT + RH) {                        // words 42 (h, last) and 43 (w, first)
        const float4 h4 = lds_f4(csH + ((RH - 1) / 2) * 16);
        rot_pair1(w[i], h4.x, h4.z);
        const float4 w4 = lds_f4(csW);
        rot_pair1(w[i + 1], w4.x, w4.z);
      } else {
        const int g = (P - RT - RH + 1) / 2;           // w record 1.. holds pairs (2g-1, 2g)
        rot_pair2(w[i], w[i + 1], lds_f4(csW + g * 16), lds_f2(nsW + g * 8));
      }
    }
    sts_u4(addr, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

// Rotate one 128-byte-swizzled row (D bf16 over D/64 panels) in place at position
// (frame, tok); or zero it when `zero` is set.  RT, RH: pairs of the t and h axes when known
// at compile time (3-D RoPE), 0 to read the split from the parameters.
template <int D, int RT, int RH>
__device__ __forceinline__ void rotate_row(uint8_t* tile, int r, int frame, int y, int x,
                                           bool zero, const float2* __restrict__ tab,
                                           const Params& p) {
  // tables are [position][pair]: a row pointer per axis plus a compile-time pair offset; the
  // w-axis rows are 21 float2 apart, so a half-warp of consecutive columns hits distinct banks
  const float2* rowT;
  const float2* rowH;
  const float2* rowW;
  if (p.rope_mode == 3) {
    rowT = tab + frame * p.rd[0];
    rowH = tab + p.tab_h_off + y * p.rd[1];
    rowW = tab + p.tab_w_off + x * p.rd[2];
  } else {
    rowT = tab + frame * (D / 2);                  // angle of frame*L_f
    rowH = tab + p.tab_h_off + (y * p.grid_w + x) * (D / 2);   // in-frame token angle
    rowW = nullptr;
  }
  const int r0 = RT > 0 ? RT : p.rd[0];
  const int r01 = RT > 0 ? RT + RH : p.rd[0] + p.rd[1];
#pragma unroll
  for (int pp = 0; pp < D / 64; ++pp) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4* ptr = reinterpret_cast<uint4*>(tile + pp * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
      if (zero) {
        *ptr = make_uint4(0, 0, 0, 0);
        continue;
      }
      uint4 v = *ptr;
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int P = pp * 32 + c * 4 + i;
        float2 cs;
        if (RT > 0) {                     // axis of pair P fixed at compile time
          cs = P < RT ? rowT[P] : (P < RT + RH ? rowH[P - RT] : rowW[P - RT - RH]);
        } else if (p.rope_mode == 3) {
          cs = P < r0 ? rowT[P] : (P < r01 ? rowH[P - r0] : rowW[P - r01]);
        } else {
          const float2 a = rowT[P], b = rowH[P];
          cs = make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
        }
        const float x0 = __uint_as_float(w[i] << 16);
        const float x1 = __uint_as_float(w[i] & 0xFFFF0000u);
        w[i] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
      }
      *ptr = v;
    }
  }
}

// RoPE tables in shared memory at `tabp`: cos / sin of pos * base^(-2j/d_axis), computed in
// double (the angle reduced exactly by sincospi) and stored as float.  RT > 0 (the 44/42/42
// split): grouped records per (axis, position, pair group): float4 (cos, cos', sin, sin') and
// float2 (-sin, -sin').  RT == 0: float2 (cos, sin) per [position][pair] (3-D: t, h, w axes;
// 1-D: the angle of the frame offset, then of the in-frame token).
template <int D, int RT, int RH>
__device__ void build_rope_tables(uint8_t* tabp, const Params& p, int tid, int nthr) {
  float4* gcs = reinterpret_cast<float4*>(tabp);            // grouped tables (RT > 0)
  float2* tab = reinterpret_cast<float2*>(tabp);             // [position][pair] (RT == 0)
  using GR = Groups<(RT > 0 ? RT : 22), (RT > 0 ? RH : 21)>;
  const int g_count = p.n_frames * GR::GT + p.grid_h * GR::GH + p.grid_w * GR::GW;
  float2* gns = reinterpret_cast<float2*>(gcs + g_count);
  if constexpr (RT > 0) {
    const int offH = p.n_frames * GR::GT, offW = offH + p.grid_h * GR::GH;
    for (int e = tid; e < g_count; e += nthr) {
      int pos, g, na;
      if (e < offH) { pos = e / GR::GT; g = e % GR::GT; na = RT; }
      else if (e < offW) { pos = (e - offH) / GR::GH; g = (e - offH) % GR::GH; na = RH; }
      else { pos = (e - offW) / GR::GW; g = (e - offW) % GR::GW; na = GR::RW; }
      double sn[2] = {0.0, 0.0}, cs[2] = {1.0, 1.0};
      const bool w_axis = e >= offW;
#pragma unroll
      for (int l = 0; l < 2; ++l) {
        // t, h: record g holds pairs (2g, 2g+1); w: record 0 holds pair 0, record g >= 1
        // holds pairs (2g-1, 2g)
        const int jj = w_axis ? (g == 0 ? (l == 0 ? 0 : na) : 2 * g - 1 + l) : 2 * g + l;
        if (jj < na) {
          const double turns = static_cast<double>(pos) *
                               exp2(-(2.0 * jj / (2 * na)) * p.log2_base) * 0.31830988618379067154;
          sincospi(turns, &sn[l], &cs[l]);
        }
      }
      gcs[e] = make_float4(static_cast<float>(cs[0]), static_cast<float>(cs[1]),
                           static_cast<float>(sn[0]), static_cast<float>(sn[1]));
      gns[e] = make_float2(-static_cast<float>(sn[0]), -static_cast<float>(sn[1]));
    }
  }
  // Layout [position][pair j]; 3-D: t (frames), h (grid rows), w (grid columns); 1-D: angle
  // of the frame offset frame*L_f, then of the in-frame token index.
  for (int e = tid; RT == 0 && e < p.tab_entries; e += nthr) {
    int pos, j, da;
    if (p.rope_mode == 3) {
      if (e < p.tab_h_off) { pos = e / p.rd[0]; j = e % p.rd[0]; da = 2 * p.rd[0]; }
      else if (e < p.tab_w_off) { const int f = e - p.tab_h_off; pos = f / p.rd[1]; j = f % p.rd[1]; da = 2 * p.rd[1]; }
      else { const int f = e - p.tab_w_off; pos = f / p.rd[2]; j = f % p.rd[2]; da = 2 * p.rd[2]; }
    } else {
      da = D;
      if (e < p.tab_h_off) { pos = (e / (D / 2)) * p.L_f; j = e % (D / 2); }
      else { const int f = e - p.tab_h_off; pos = f / (D / 2); j = f % (D / 2); }
    }
    // angle / pi, so that the reduction of the argument is exact (sincospi)
    const double turns = static_cast<double>(pos) * exp2(-(2.0 * j / da) * p.log2_base) *
                         0.31830988618379067154;
    double sn, cs;
    sincospi(turns, &sn, &cs);
    tab[e] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
}

// kFused = false: every key from the slot-indexed raw caches (tm_k, tm_v), rotated here.
// kFused = true: keys of every slot but the current block's from the rotated copy (tm_k =
// k_rot, already rotated at this block's positions; tm_v = v_cache); the current block's keys
// and values from k_new / v_new (tm_kn, tm_vn), rotated here, and also stored raw into their
// ring slot (tm_ks, tm_vs: maps over that slot of k_cache / v_cache), each tile by one CTA.
template <int D, int RT, int RH, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
prsink_attention_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_kn,
                        const __grid_constant__ CUtensorMap tm_vn,
                        const __grid_constant__ CUtensorMap tm_ks,
                        const __grid_constant__ CUtensorMap tm_vs,
                        const __grid_constant__ CUtensorMap tm_o, const Params p) {
  using LY = Layout<D>;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[B_COUNT];
  __shared__ uint32_t tmem_base_s;
  __shared__ AbortState ab;
  __shared__ unsigned vmask_s;
  __shared__ uint16_t tile_list[kMaxTiles];      // live tiles in order (kTile* bits)
  __shared__ int n_live_s;
  __shared__ int last_k_s, last_v_s;             // last K / V loads issued (for the drain)
  __shared__ int list_off_s;                     // first tile of this CTA's share
  __shared__ int combine_s;                      // this CTA combines the split partials

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t sb = (raw + 1023u) & ~1023u;            // 1 KB aligned base (swizzle atoms)
  uint8_t* gb = dsmem + (sb - raw);
  const uint32_t sQ = sb + LY::kQ, sK = sb + LY::kK, sV = sb + LY::kV;
  float2* tab = reinterpret_cast<float2*>(gb + LY::kTab);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  int unit = blockIdx.x, split = 0, n_split = 1;
  if (unit >= p.split_base) {
    const int k = unit - p.split_base;
    n_split = p.n_split;
    unit = p.split_base + k / n_split;
    split = k % n_split;
  }
  const int h = unit / p.nqb, qb = unit % p.nqb;
  const int q0 = qb * (NQ * BM);

  if (threadIdx.x == 32) {
    // warp 1: the barriers, then Q, which needs no tile list, goes out at once
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QREADY), NQ * BM);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KREADY + s), 128);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VFIX + s), 128);
      mbar_init(bar(B_VEMPTY + s), 1);
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_PFULL + s), 128);
      mbar_init(bar(B_ODONE + s), 1);
    }
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_KSTORED + 0), 1);
    mbar_init(bar(B_KSTORED + 1), 1);
    ab.flag = 0;
    last_k_s = last_v_s = -1;
    fence_barrier_init();
    mbar_arrive_expect_tx(bar(B_QFULL), NQ * LY::kTileBytes);
    for (int qt = 0; qt < NQ; ++qt)
      for (int pp = 0; pp < D / 64; ++pp)
        tma_load_3d(sQ + qt * LY::kTileBytes + pp * 16384, &tm_q, bar(B_QFULL), pp * 64, h,
                    q0 + qt * BM);
  }
  if (threadIdx.x == 0) {
    // warp 0: the slots this call attends to, for its tile list below
    unsigned vm = p.valid_mask;
    if (p.dyn_src && *p.dyn_src < 0) vm &= ~(1u << PRSINK_SLOT_DYNAMIC);
    if (kFused) vm &= ~(1u << p.cur_slot);        // its keys come from k_new instead
    vmask_s = vm;
  }
  const int n_tiles = (p.T + BN - 1) / BN;
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (kFused) {
      prefetch_tmap(&tm_kn);
      prefetch_tmap(&tm_vn);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&tmem_base_s), kTmemCols);
    tmem_relinquish();
  }
  // RoPE tables (cos / sin in shared memory).  The fused form builds them after the prologue's
  // barrier, while the first loads are in flight; the unfused form here, before it (measured on a
  // B200: each placement is 1.5-5 % slower in the other form)
  float4* gcs = reinterpret_cast<float4*>(gb + LY::kTab);   // grouped tables (RT > 0)
  using GR = Groups<(RT > 0 ? RT : 22), (RT > 0 ? RH : 21)>;
  float2* gns = reinterpret_cast<float2*>(
      gcs + (p.n_frames * GR::GT + p.grid_h * GR::GH + p.grid_w * GR::GW));
  if constexpr (!kFused) build_rope_tables<D, RT, RH>(gb + LY::kTab, p, threadIdx.x, kThreads);
  if (warp == 0) {
    __syncwarp();                                  // vmask_s from lane 0
    // the tiles holding a valid key (boundary tiles flagged for masking), 32 at a time, in order
    const unsigned vm0 = vmask_s;
    const SlotBounds sbnd(p);
    int base = 0;
    for (int n0 = 0; n0 < n_tiles; n0 += 32) {
      const int n = n0 + lane;
      const int f = n < n_tiles ? sbnd.flags(n, vm0, p) : 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, f & 1);
      if (f & 1)
        tile_list[base + __popc(bal & ((1u << lane) - 1u))] =
            static_cast<uint16_t>(n | ((f & 2) ? (kTileMask | kTileVfix) : 0));
      base += __popc(bal);
    }
    if (kFused) {
      // the current block's tiles after the sink tiles; tile i is stored by the CTA of query
      // pair i mod nqb
      for (int i = lane; i < p.n_cur_tiles; i += 32) {
        uint16_t e = static_cast<uint16_t>(i) | kTileNew;
        if ((i + 1) * BN > p.L_blk) e |= kTileMask;
        if (i % p.nqb == qb)
          e |= kTileStore | kTileVfix;
        tile_list[base + i] = e;
      }
      base += p.n_cur_tiles;
    }
    if (lane == 0) {
      // a split CTA takes an equal share of the live tiles
      const int j0 = static_cast<int>(static_cast<long long>(base) * split / n_split);
      const int j1 = static_cast<int>(static_cast<long long>(base) * (split + 1) / n_split);
      list_off_s = j0;
      n_live_s = j1 - j0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const unsigned vm = vmask_s;
  const uint64_t deadline = globaltimer() + p.timeout_ns;
  const int n_live = n_live_s;
  const uint16_t* tiles = tile_list + list_off_s;

  // TMA loads of tile j's K and V into stage j & 1 (tiles j >= 2 first wait for the stage to be
  // released); false when a wait gave up
  auto load_kv = [&](int j) -> bool {
    const uint16_t te = tiles[j];
    const int n = te & kTileIdx;
    const bool cur = kFused && (te & kTileNew);    // [tokens][H][d] map: (d, head, token)
    const int c1 = cur ? h : n * BN, c2 = cur ? n * BN : h;
    const int st = j & 1;
    const uint32_t par = ((j >> 1) - 1) & 1;
    if (j >= 2 && !mbar_wait(bar(B_KEMPTY + st), par, &ab, deadline, p.status)) return false;
    mbar_arrive_expect_tx(bar(B_KFULL + st), LY::kTileBytes);
    for (int pp = 0; pp < D / 64; ++pp)
      tma_load_3d(sK + st * LY::kTileBytes + pp * 16384, cur ? &tm_kn : &tm_k,
                  bar(B_KFULL + st), pp * 64, c1, c2);
    last_k_s = j;
    if (j >= 2 && !mbar_wait(bar(B_VEMPTY + st), par, &ab, deadline, p.status)) return false;
    mbar_arrive_expect_tx(bar(B_VFULL + st), LY::kTileBytes);
    for (int pp = 0; pp < D / 64; ++pp)
      tma_load_3d(sV + st * LY::kTileBytes + pp * 16384, cur ? &tm_vn : &tm_v,
                  bar(B_VFULL + st), pp * 64, c1, c2);
    last_v_s = j;
    return true;
  };
  // the producer sends the first two K/V tiles out at once (their stages are free, so nothing
  // waits)
  if (warp == kProducerWarp && lane == 0)
    for (int j = 0; j < 2 && j < n_live; ++j) load_kv(j);
  if constexpr (kFused) {
    build_rope_tables<D, RT, RH>(gb + LY::kTab, p, threadIdx.x, kThreads);
    __syncthreads();
  }

  if (warp >= kProducerWarp) {
    setmaxnreg_dec<80>();
    if (warp == kProducerWarp && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      // (Q and tiles 0, 1 are already on their way)
      for (int j = 2; j < n_live; ++j)
        if (!load_kv(j)) break;
    } else if (warp == kMmaWarp && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(bar(B_QREADY), 0, &ab, deadline, p.status);
      tc_fence_after();
      int fix0 = 0, fix1 = 0;                              // boundary tiles seen per stage
      // base descriptors, computed once: Q0, Q1, the two K stages and the two V stages
      const uint64_t dq0 = sdesc_sw128(sQ, 16, 1024), dq1 = sdesc_sw128(sQ + LY::kTileBytes, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024), dk1 = sdesc_sw128(sK + LY::kTileBytes, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, 16384, 1024), dv1 = sdesc_sw128(sV + LY::kTileBytes, 16384, 1024);
      auto s_mma = [&](int qt, int st) {
        const uint64_t a = qt ? dq1 : dq0, b = st ? dk1 : dk0;
        if constexpr (D == 128) umma_ss_k128(tmem + LY::col_s(qt), a, b, LY::kIdescS);
        else umma_ss_k64(tmem + LY::col_s(qt), a, b, LY::kIdescS);
      };
      // O_qt (+)= P_qt(i) V(i); V(i) must have landed (and been fixed up in boundary tiles)
      auto pv_mma = [&](int qt, int i, bool partial) -> bool {
        const int st = i & 1;
        if (qt == 0) {
          if (!mbar_wait(bar(B_VFULL + st), (i >> 1) & 1, &ab, deadline, p.status)) return false;
          if (partial) {
            int& fx = st ? fix1 : fix0;
            if (!mbar_wait(bar(B_VFIX + st), fx & 1, &ab, deadline, p.status)) return false;
            ++fx;
          }
        }
        if (!mbar_wait(bar(B_PFULL + qt), i & 1, &ab, deadline, p.status)) return false;
        tc_fence_after();
        umma_ts_pv128(tmem + LY::col_o(qt), tmem + LY::col_s(qt), st ? dv1 : dv0, LY::kIdescPV,
                      i > 0 ? 1u : 0u);
        return true;
      };
      int j = 0;
      bool prev_partial = false;
      int kready0 = 0, kready1 = 0;            // K tiles handed over by the rotation warps
      for (; ok && j < n_live; ++j) {
        const uint16_t te = tiles[j];
        const bool partial = te & kTileVfix;              // V touched by the rotation warps
        const int st = j & 1;
        // P0(j-1).V(j-1) does not need K(j): issue it before waiting for the rotation
        if (j >= 1 && !pv_mma(0, j - 1, prev_partial)) { ok = false; break; }
        // fused form: a tile of the rotated copy goes to the tensor core as it landed
        const bool direct = kFused && !(te & kTileNew);
        const uint32_t kbar = direct ? bar(B_KFULL + st) : bar(B_KREADY + st);
        const uint32_t kpar = direct ? ((j >> 1) & 1) : ((st ? kready1++ : kready0++) & 1);
        if (!mbar_wait(kbar, kpar, &ab, deadline, p.status)) { ok = false; break; }
        tc_fence_after();
        s_mma(0, st);
        // self-test of the abort path: without this commit the softmax of tile 0 waits until
        // its deadline, raises the abort flag and every role drains and exits
        if (!(p.debug_stall && j == 0)) umma_commit(bar(B_SFULL + 0));
        if (j >= 1) {
          if (!pv_mma(1, j - 1, prev_partial)) { ok = false; break; }
          umma_commit(bar(B_VEMPTY + ((j - 1) & 1)));
        }
        s_mma(1, st);
        umma_commit(bar(B_SFULL + 1));
        umma_commit(bar(B_KEMPTY + st));
        prev_partial = partial;
      }
      if (ok && j >= 1) {
        if (pv_mma(0, j - 1, prev_partial)) {
          umma_commit(bar(B_ODONE + 0));
          if (pv_mma(1, j - 1, prev_partial)) {
            umma_commit(bar(B_VEMPTY + ((j - 1) & 1)));
            umma_commit(bar(B_ODONE + 1));
          }
        }
      }
    }
  } else if (warp >= kRotWarp0) {
    // ------------------------------------------------------------------ rotation
    setmaxnreg_dec<64>();
    const int rt = threadIdx.x - kRotWarp0 * 32;          // row of the tile, 0..127
    {   // (Q is rotated by the softmax warps, one query row per thread)
      // position of this thread's key row, advanced incrementally from tile to tile
      int cur = -2 * BN, s_cur = 0, frame = 0, y = 0, x = 0;   // no previous row yet
      // raw K tiles stored so far, per stage: a stage is reloaded only after all 128 threads
      // handed over its previous tile, so the store barrier of a stage never runs two phases
      // ahead of a thread that still has to see its last phase
      int n_stored0 = 0, n_stored1 = 0;
      for (int j = 0; j < n_live; ++j) {
        const uint16_t te = tiles[j];
        const int n = te & kTileIdx;
        const int st = j & 1;
        const uint32_t kt = sK + st * LY::kTileBytes;
        if (kFused && !(te & kTileNew)) {
          // a tile of the rotated copy: the MMA reads K as it landed; only the V rows of empty
          // slots in a boundary tile need zeroing here.  The K wait still comes first, for
          // every tile in order: a parity wait is only sound for a waiter at most one phase
          // ahead, and skipping tiles would let these warps run further ahead than that.
          if (!mbar_wait(bar(B_KFULL + st), (j >> 1) & 1, &ab, deadline, p.status)) break;
          if (te & kTileVfix) {
            const int row = n * BN + rt;
            const bool empty = row < p.T && !((vm >> slot_of(row, p)) & 1u);
            if (!mbar_wait(bar(B_VFULL + st), (j >> 1) & 1, &ab, deadline, p.status)) break;
            if (empty)
              rotate_row<D, RT, RH>(gb + LY::kV + st * LY::kTileBytes, rt, 0, 0, 0, true, tab, p);
            fence_proxy_async_smem();
            mbar_arrive(bar(B_VFIX + st));
          }
          continue;
        }
        if (!mbar_wait(bar(B_KFULL + st), (j >> 1) & 1, &ab, deadline, p.status)) break;
        bool empty = false;
        if (kFused && (te & kTileNew)) {
          // the current block: store the raw tile into its ring slot (one CTA per tile), then
          // rotate it at the current block's positions
          if (te & kTileStore) {
            if (rt == 0) {
              for (int pp = 0; pp < D / 64; ++pp)
                tma_store_3d(&tm_ks, kt + pp * 16384, pp * 64, n * BN, h);
              bulk_commit();
              bulk_wait_read_all();
              mbar_arrive(bar(B_KSTORED + st));
            }
            const int ns = st ? n_stored1++ : n_stored0++;
            if (!mbar_wait(bar(B_KSTORED + st), ns & 1, &ab, deadline, p.status)) break;
          }
          const int ti = n * BN + rt;
          if (ti < p.L_blk) {
            const int tok = ti % p.L_f;
            if constexpr (RT > 0)
              rotate_row_grouped<RT, RH>(kt, rt, p.q_frame + ti / p.L_f, tok / p.grid_w,
                                         tok % p.grid_w, false, smem_u32(gcs), smem_u32(gns), p);
            else
              rotate_row<D, RT, RH>(gb + LY::kK + st * LY::kTileBytes, rt, p.q_frame + ti / p.L_f,
                                    tok / p.grid_w, tok % p.grid_w, false, tab, p);
          }
        } else {
          const int row = n * BN + rt;
          if (row < p.T) {
            if (row == cur + BN && row < p.slot_start[s_cur + 1]) {
              x += p.step_x;                       // one tile further in the same slot
              y += p.step_y;
              if (x >= p.grid_w) { x -= p.grid_w; ++y; }
              while (y >= p.grid_h) { y -= p.grid_h; ++frame; }
            } else {
              s_cur = slot_of(row, p);
              const int u = row - p.slot_start[s_cur];
              const int tok = u % p.L_f;
              frame = p.slot_frame[s_cur] + u / p.L_f;
              y = tok / p.grid_w;
              x = tok - y * p.grid_w;
            }
            cur = row;
            empty = !((vm >> s_cur) & 1u);
            if constexpr (RT > 0)
              rotate_row_grouped<RT, RH>(kt, rt, frame, y, x, empty, smem_u32(gcs),
                                         smem_u32(gns), p);
            else
              rotate_row<D, RT, RH>(gb + LY::kK + st * LY::kTileBytes, rt, frame, y, x, empty,
                                    tab, p);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_KREADY + st));
        if (te & kTileVfix) {
          // boundary tile: empty-slot rows of V may hold anything; P is 0 there, but 0 * NaN
          // is not, so zero them before the P.V MMA reads the tile.  A current-block tile this
          // CTA stores: its raw V goes to the ring slot before the P.V MMA may release it.
          if (!mbar_wait(bar(B_VFULL + st), (j >> 1) & 1, &ab, deadline, p.status)) break;
          if (kFused && (te & kTileStore)) {
            if (rt == 0) {
              for (int pp = 0; pp < D / 64; ++pp)
                tma_store_3d(&tm_vs, sV + st * LY::kTileBytes + pp * 16384, pp * 64, n * BN, h);
              bulk_commit();
              bulk_wait_read_all();
            }
          } else if (empty) {
            rotate_row<D, RT, RH>(gb + LY::kV + st * LY::kTileBytes, rt, 0, 0, 0, true, tab, p);
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(B_VFIX + st));
        }
      }
      if (kFused && rt == 0) bulk_wait_all();    // the ring-slot stores complete before exit
    }
  } else {
    // ------------------------------------------------------------------ softmax (warps 0-7)
    setmaxnreg_inc<184>();
    const int qt = warp >> 2;                             // query tile of this warpgroup
    const int t = threadIdx.x & (BM - 1);                 // query row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + LY::col_s(qt);
    const uint32_t tO = tmem + lane_off + LY::col_o(qt);
    const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
    float m = -INFINITY, l = 0.f;
    int j = 0;
    // this thread's own query row, rotated at its position while the rotation warps take the
    // first key tiles
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_QFULL), 0, &ab, deadline, p.status));
    if (ok) {
      const int qi = q0 + qt * BM + t;
      if (qi < p.L_blk) {
        const int tok = qi % p.L_f;
        if constexpr (RT > 0)
          rotate_row_grouped<RT, RH>(sQ + qt * LY::kTileBytes, t, p.q_frame + qi / p.L_f,
                                     tok / p.grid_w, tok % p.grid_w, false, smem_u32(gcs),
                                     smem_u32(gns), p);
        else
          rotate_row<D, RT, RH>(gb + LY::kQ + qt * LY::kTileBytes, t, p.q_frame + qi / p.L_f,
                                tok / p.grid_w, tok % p.grid_w, false, tab, p);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(B_QREADY));
    }
    for (; ok && j < n_live; ++j) {
      const uint16_t te = tiles[j];
      const int n = te & kTileIdx;
      ok = mbar_wait(bar(B_SFULL + qt), j & 1, &ab, deadline, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }   // tcgen05.ld is warp-collective
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_wait_ld();
      if (te & kTileMask) {
        // columns of empty slots and past the end of the cache (or, for the current block's
        // last tile, past its last token): 4 mask words, built per slot
        const int lo = n * BN;
        uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};
        const bool cur_tile = kFused && (te & kTileNew);
        for (int s2 = cur_tile ? p.n_slots : 0; s2 <= p.n_slots; ++s2) {
          int a, e;
          if (cur_tile) {
            a = p.L_blk - lo;
            e = BN;
          } else if (s2 < p.n_slots) {
            if ((vm >> s2) & 1u) continue;
            a = p.slot_start[s2] - lo;
            e = p.slot_start[s2 + 1] - lo;
          } else {
            a = p.T - lo;
            e = BN;
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int cl = max(a, w * 32), ch = min(e, w * 32 + 32);
            if (cl < ch) {
              const uint32_t bits = (ch - cl == 32) ? ~0u : (((1u << (ch - cl)) - 1u) << (cl - w * 32));
              mw[w] &= ~bits;
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = __float_as_uint(-INFINITY);
      }
      // row max of the raw scores (scaling by a positive constant keeps the argmax); eight
      // independent partial maxima keep the dependency chains short
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = __uint_as_float(s[a]);
      if constexpr (kMax3) {
#pragma unroll
        for (int c = 8; c < 120; c += 16)
#pragma unroll
          for (int a = 0; a < 8; ++a)
            mx[a] = fmax3(mx[a], __uint_as_float(s[c + a]), __uint_as_float(s[c + 8 + a]));
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmaxf(mx[a], __uint_as_float(s[120 + a]));
      } else {
#pragma unroll
        for (int c = 8; c < 128; c += 8)
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = fmaxf(mx[a], __uint_as_float(s[c + a]));
      }
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = mt;
      } else if (mt > m + kRescaleThreshold) {
        alpha = ex2(m - mt);
        m = mt;
        rescale = true;
      }
      if (__any_sync(0xffffffffu, rescale)) {   // rows that keep their max scale by alpha = 1
        // O_qt holds every P.V up to tile j-1 (the S(j) commit completed after them); it is
        // rescaled before P of tile j is written (measured no slower than after it)
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
      }
      // P = 2^(s*scale - m) as bf16 pairs into the S columns (A operand of the P.V MMA):
      // 32 scores -> 16 packed words -> one 16-column TMEM store
      const float2 negm = make_float2(-m, -m);
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};               // independent partial sums
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = ch * 32 + 2 * i;
          const float2 e2 = ffma2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                  scale2, negm);
          const float2 pr = ((kPolyPairs >> i) & 1u) ? exp2_poly2(e2)
                                                      : make_float2(ex2(e2.x), ex2(e2.y));
          sum2[i & 3] = fadd2(sum2[i & 3], pr);
          pk[i] = pack_bf16(pr.x, pr.y);
        }
        tmem_st16(tS + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + qt));
      const float2 s01 = fadd2(sum2[0], sum2[1]), s23 = fadd2(sum2[2], sum2[3]);
      const float2 s4 = fadd2(s01, s23);
      l = l * alpha + (s4.x + s4.y);
    }
    // epilogue: O / l -> bf16.  A whole unit stages its rows in the tile's own Q buffer (free:
    // ODONE follows every S MMA), in the layout the Q load used (128-byte swizzled panels of 64
    // columns), and one thread stores the tile with TMA (rows past the block are clipped); a
    // split CTA writes its unnormalised float32 partial row (O, max, sum) for the combine.
    const int qi = q0 + qt * BM + t;
    float inv = 0.f;
    bool have = false;
    if (__all_sync(0xffffffffu, ok) && j > 0) {
      have = mbar_wait(bar(B_ODONE + qt), 0, &ab, deadline, p.status);
      have = __all_sync(0xffffffffu, have);
      tc_fence_after();
      inv = l > 0.f ? 1.f / l : 0.f;
    }
    const uint32_t so = sQ + qt * LY::kTileBytes;
    const size_t slot = static_cast<size_t>(unit - p.split_base) * n_split + split;
    float* prow = n_split > 1 ? p.part_o + (slot * (NQ * BM) + qt * BM + t) * D : nullptr;
    if (n_split > 1)
      p.part_ml[slot * (NQ * BM) + qt * BM + t] =
          have ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      if (have) {                     // warp-uniform
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (prow) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<uint4*>(prow + cc * 32 + i) = make_uint4(o[i], o[i + 1], o[i + 2],
                                                                     o[i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
          const int k = (cc * 32 + i) >> 3;           // 16-byte chunk of the row
          sts_u4(so + (k >> 3) * 16384 + t * 128 + (((k & 7) ^ (t & 7)) << 4), v);
        }
      }
    }
    if (!prow) {
      fence_proxy_async_smem();
      named_bar_sync(1 + qt, BM);                     // the tile's 128 rows are staged
      if (t == 0) {
        for (int pp = 0; pp < D / 64; ++pp)
          tma_store_3d(&tm_o, so + pp * 16384, pp * 64, h, q0 + qt * BM);
        bulk_commit();
        bulk_wait_all();                              // complete before the CTA exits
      }
    }
    if (p.lse && qi < p.L_blk && n_split == 1)
      p.lse[static_cast<size_t>(h) * p.L_blk + qi] =
          have ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    if (n_split > 1) __threadfence();   // partials visible before this CTA's arrival counts
  }

  tc_fence_before();
  __syncthreads();
  // Every role has left its loop, so the abort flag is final here.  After an abort, copies and
  // MMAs may still be in flight: let them complete before the CTA's shared and tensor memory
  // are released (bounded waits; an abort raised late by one role is seen by all).
  if (ab.flag) {
    if (warp == kProducerWarp && lane == 0) {
      drain_wait(bar(B_QFULL), 0, 100000000ull);
      for (int i = last_k_s - 1; i <= last_k_s; ++i)
        if (i >= 0) drain_wait(bar(B_KFULL + (i & 1)), (i >> 1) & 1, 100000000ull);
      for (int i = last_v_s - 1; i <= last_v_s; ++i)
        if (i >= 0) drain_wait(bar(B_VFULL + (i & 1)), (i >> 1) & 1, 100000000ull);
    }
    if (warp == kMmaWarp && lane == 0) {       // the thread that issued every MMA
      umma_commit(bar(B_FINAL));
      drain_wait(bar(B_FINAL), 0, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (n_split > 1) {
    // the last of a unit's split CTAs to arrive combines their partials:
    //   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  O = sum_s O_s 2^(m_s - M) / L
    const size_t k = static_cast<size_t>(unit - p.split_base);
    if (threadIdx.x == 0) {
      __threadfence();
      combine_s = atomicAdd(&p.part_cnt[k], 1) == n_split - 1;
    }
    __syncthreads();
    if (combine_s) {
      __threadfence();
      const int r = threadIdx.x;                  // one row per thread
      const int qi = q0 + r;
      if (r < NQ * BM && qi < p.L_blk) {
        const float2* ml = p.part_ml + k * n_split * (NQ * BM) + r;
        float M = -INFINITY;
        for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, __ldcg(ml + sp * (NQ * BM)).x);
        // weight of share sp: 2^(m_s - M), 0 for a share without keys (or no keys at all)
        auto weight = [&](int sp) {
          const float ms = __ldcg(ml + sp * (NQ * BM)).x;
          return ms > -INFINITY ? ex2(ms - M) : 0.f;
        };
        float L = 0.f;
        for (int sp = 0; sp < n_split; ++sp) L += weight(sp) * __ldcg(ml + sp * (NQ * BM)).y;
        const float inv = L > 0.f ? 1.f / L : 0.f;
        __nv_bfloat16* orow = p.out + (static_cast<size_t>(qi) * p.H + h) * D;
        const float* o0 = p.part_o + (k * n_split * (NQ * BM) + r) * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 8) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int sp = 0; sp < n_split; ++sp) {
            const float w = weight(sp);
            const float4* src =
                reinterpret_cast<const float4*>(o0 + static_cast<size_t>(sp) * (NQ * BM) * D + c);
            const float4 a = __ldcg(src), b = __ldcg(src + 1);
            acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
            acc[4] += w * b.x; acc[5] += w * b.y; acc[6] += w * b.z; acc[7] += w * b.w;
          }
          uint4 v;
          v.x = pack_bf16(acc[0] * inv, acc[1] * inv);
          v.y = pack_bf16(acc[2] * inv, acc[3] * inv);
          v.z = pack_bf16(acc[4] * inv, acc[5] * inv);
          v.w = pack_bf16(acc[6] * inv, acc[7] * inv);
          *reinterpret_cast<uint4*>(orow + c) = v;
        }
        if (p.lse)
          p.lse[static_cast<size_t>(h) * p.L_blk + qi] =
              L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
      }
      if (threadIdx.x == 0) p.part_cnt[k] = 0;   // ready for the next launch
    }
  }
}

// ---------------------------------------------------------------------------- rotation pass
// prsink_rotate_sinks: the raw keys of the slots in the rotation mask rotated at this block's
// positions into k_rot (same [H][T][d] layout), with the attention kernel's own rotation code,
// so that the fused attention reads keys bitwise equal to the ones it would rotate itself.
// Work item = (head, key tile of 128 rows).  A CTA (one per SM) runs kRotGroups independent
// 128-thread pipelines that share one copy of the RoPE tables; each streams its items through
// its own two shared-memory stages: TMA load of the raw tile, one row per thread rotated in
// place, TMA store.  Rows of other slots that share a boundary tile are rotated and stored too:
// their rotated copies are either rewritten identically (slots whose positions are fixed) or
// never read.
constexpr int kRotGroups = 3;
constexpr int kRotThreads = 128 * kRotGroups;

template <int D, int RT, int RH>
__global__ void __launch_bounds__(kRotThreads)
prsink_rotate_kernel(const __grid_constant__ CUtensorMap tm_src,
                     const __grid_constant__ CUtensorMap tm_dst, const Params p) {
  using LY = Layout<D>;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full[kRotGroups][2];
  __shared__ AbortState ab;
  __shared__ unsigned mask_s;
  __shared__ uint16_t tile_list[kMaxTiles];
  __shared__ int n_live_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = threadIdx.x >> 7, rt = threadIdx.x & 127;   // pipeline, row of the tile
  const bool leader = rt == 0;
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = dsmem + (sb - raw);
  const uint32_t stage0 = sb + grp * 2 * LY::kTileBytes;      // this pipeline's two stages
  constexpr int kTabOff = kRotGroups * 2 * LY::kTileBytes;
  if (threadIdx.x == 0) {
    for (int g = 0; g < kRotGroups; ++g) {
      mbar_init(smem_u32(&full[g][0]), 1);
      mbar_init(smem_u32(&full[g][1]), 1);
    }
    ab.flag = 0;
    unsigned m = p.rot_mask & p.valid_mask;
    if (p.cur_slot >= 0) m &= ~(1u << p.cur_slot);
    if ((p.dyn_src && *p.dyn_src < 0) || (p.rot_dyn_flag && *p.rot_dyn_flag == 0))
      m &= ~(1u << PRSINK_SLOT_DYNAMIC);
    mask_s = m;
    fence_barrier_init();
  }
  if (warp == 0) {
    __syncwarp();                                  // mask_s from lane 0
    const int n_tiles = (p.T + BN - 1) / BN;
    const unsigned m = mask_s;
    const SlotBounds sbnd(p);
    int base = 0;
    for (int n0 = 0; n0 < n_tiles; n0 += 32) {
      const int n = n0 + lane;
      const bool live = n < n_tiles && (sbnd.flags(n, m, p) & 1);
      const uint32_t bal = __ballot_sync(0xffffffffu, live);
      if (live) tile_list[base + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(n);
      base += __popc(bal);
    }
    if (lane == 0) n_live_s = base;
  }
  __syncthreads();
  const int n_live = n_live_s;
  const int total = n_live * p.H;
  const int stride = gridDim.x * kRotGroups;
  const int w0 = blockIdx.x * kRotGroups + grp;
  const uint64_t deadline = globaltimer() + p.timeout_ns;
  auto item = [&](int w, int& n, int& h) { h = w / n_live; n = tile_list[w - h * n_live]; };
  auto load = [&](int w, int st) {
    int n, h;
    item(w, n, h);
    const uint32_t bar = smem_u32(&full[grp][st]);
    mbar_arrive_expect_tx(bar, LY::kTileBytes);
    for (int pp = 0; pp < D / 64; ++pp)
      tma_load_3d(stage0 + st * LY::kTileBytes + pp * 16384, &tm_src, bar, pp * 64, n * BN, h);
  };
  // each pipeline's first load goes out before the RoPE tables are built
  int i = 0, last_load = -1;
  if (leader && w0 < total) {
    prefetch_tmap(&tm_src);
    prefetch_tmap(&tm_dst);
    load(w0, 0);
    last_load = 0;
  }
  float4* gcs = reinterpret_cast<float4*>(gb + kTabOff);
  using GR = Groups<(RT > 0 ? RT : 22), (RT > 0 ? RH : 21)>;
  float2* gns = reinterpret_cast<float2*>(
      gcs + (p.n_frames * GR::GT + p.grid_h * GR::GH + p.grid_w * GR::GW));
  float2* tab = reinterpret_cast<float2*>(gb + kTabOff);
  build_rope_tables<D, RT, RH>(gb + kTabOff, p, threadIdx.x, kRotThreads);
  __syncthreads();
  for (int w = w0; w < total; w += stride, ++i) {
    const int st = i & 1;
    const int wn = w + stride;
    if (leader && wn < total) {
      bulk_wait_read_all();             // the store of item i-1 has read stage st^1
      load(wn, st ^ 1);
      last_load = i + 1;
    }
    // every thread of the pipeline takes the same decision (a wait that gave up in one thread
    // ends the loop for all, so no thread is left behind at the barrier below)
    if (!named_bar_and(1 + grp, 128, mbar_wait(smem_u32(&full[grp][st]), (i >> 1) & 1, &ab,
                                                deadline, p.status)))
      break;
    int n, h;
    item(w, n, h);
    const int row = n * BN + rt;
    if (row < p.T) {
      const int s = slot_of(row, p);
      const int u = row - p.slot_start[s];
      const int tok = u % p.L_f;
      const int frame = p.slot_frame[s] + u / p.L_f;
      if constexpr (RT > 0)
        rotate_row_grouped<RT, RH>(stage0 + st * LY::kTileBytes, rt, frame, tok / p.grid_w,
                                   tok % p.grid_w, false, smem_u32(gcs), smem_u32(gns), p);
      else
        rotate_row<D, RT, RH>(gb + (stage0 - sb) + st * LY::kTileBytes, rt, frame,
                              tok / p.grid_w, tok % p.grid_w, false, tab, p);
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + grp, 128);
    if (leader) {
      for (int pp = 0; pp < D / 64; ++pp)
        tma_store_3d(&tm_dst, stage0 + st * LY::kTileBytes + pp * 16384, pp * 64, n * BN, h);
      bulk_commit();
    }
  }
  if (leader) {
    if (ab.flag) {                      // let loads in flight land before shared memory goes
      for (int k = last_load - 1; k <= last_load; ++k)
        if (k >= i) drain_wait(smem_u32(&full[grp][k & 1]), (k >> 1) & 1, 100000000ull);
    }
    bulk_wait_all();
  }
}

// ---------------------------------------------------------------------------- host side
// Device buffers of one call: q, the key / value sources of the slot-indexed tiles (raw caches,
// or k_rot and v_cache in the fused form), and for the fused form k_new, v_new and the caches
// whose current ring slot receives the raw block.
struct Buffers {
  const void* q;
  const void* k;
  const void* v;
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
};

static int table_bytes(const prsink_layout* L, const Params& p, bool grouped) {
  using GR = Groups<22, 21>;
  return grouped ? (p.n_frames * GR::GT + L->grid_h * GR::GH + L->grid_w * GR::GW) * 24
                 : p.tab_entries * 8;
}

// Allow `smem` bytes of dynamic shared memory for `fn` (once per size and device).
template <typename F>
static int allow_smem(F fn, int smem, int (&allowed)[64], const char* what) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (allowed[dev] < smem) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return check_launch(what);
    allowed[dev] = smem;
  }
  return PRSINK_OK;
}

template <int D, int RT, int RH, bool kFused>
static int launch(const prsink_layout* L, const Geometry& g, const Buffers& b, Params& p,
                  cudaStream_t st) {
  const char* what = kFused ? "prsink_attention_fused" : "prsink_attention";
  const uint64_t H = L->n_heads;
  CUtensorMap mq, mk, mv, mkn, mvn, mks, mvs, mo;
  int rc = make_map(&mq, b.q, D, H, g.L_blk, 2ull * D, 2ull * D * H, 1, BM);
  // the output has Q's layout ([L_blk][H][d]); whole tiles leave through TMA stores
  if (!rc) rc = make_map(&mo, p.out, D, H, g.L_blk, 2ull * D, 2ull * D * H, 1, BM);
  if (!rc) rc = make_map(&mk, b.k, D, g.T, H, 2ull * D, 2ull * D * g.T, BN, 1);
  if (!rc) rc = make_map(&mv, b.v, D, g.T, H, 2ull * D, 2ull * D * g.T, BN, 1);
  if (kFused) {
    // current block: token-major k_new / v_new; raw store: the ring slot's rows of the caches
    const uint64_t off = 2ull * D * static_cast<uint64_t>(g.slot_start[p.cur_slot]);
    if (!rc) rc = make_map(&mkn, b.k_new, D, H, g.L_blk, 2ull * D, 2ull * D * H, 1, BN);
    if (!rc) rc = make_map(&mvn, b.v_new, D, H, g.L_blk, 2ull * D, 2ull * D * H, 1, BN);
    if (!rc) rc = make_map(&mks, static_cast<char*>(b.k_cache) + off, D, g.L_blk, H, 2ull * D,
                           2ull * D * g.T, BN, 1);
    if (!rc) rc = make_map(&mvs, static_cast<char*>(b.v_cache) + off, D, g.L_blk, H, 2ull * D,
                           2ull * D * g.T, BN, 1);
  } else {
    mkn = mvn = mks = mvs = mk;                 // unused
  }
  if (rc) return rc;
  const int tab = table_bytes(L, p, RT > 0);
  if (tab > kTableMaxBytes) {
    set_error("%s: RoPE tables need %d bytes of shared memory (max %d)", what, tab,
              kTableMaxBytes);
    return PRSINK_ERR_UNSUPPORTED;
  }
  int smem = Layout<D>::kTab + tab + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;     // one CTA per SM (it holds all 512 TMEM columns)
  static int allowed[64] = {0};
  rc = allow_smem(prsink_attention_kernel<D, RT, RH, kFused>, smem, allowed, what);
  if (rc) return rc;
  const int units = p.nqb * L->n_heads;
  const int ctas = p.split_base + (units - p.split_base) * p.n_split;
  prsink_attention_kernel<D, RT, RH, kFused><<<ctas, kThreads, smem, st>>>(mq, mk, mv, mkn, mvn,
                                                                          mks, mvs, mo, p);
  count_launch();
  return check_launch(what);
}

template <int D, int RT, int RH>
static int launch_rotate(const prsink_layout* L, const Geometry& g, const void* k_cache,
                         void* k_rot, Params& p, cudaStream_t st) {
  const uint64_t H = L->n_heads;
  CUtensorMap ms, md;
  int rc = make_map(&ms, k_cache, D, g.T, H, 2ull * D, 2ull * D * g.T, BN, 1);
  if (!rc) rc = make_map(&md, k_rot, D, g.T, H, 2ull * D, 2ull * D * g.T, BN, 1);
  if (rc) return rc;
  const int tab = table_bytes(L, p, RT > 0);
  if (tab > kTableMaxBytes) {
    set_error("prsink_rotate_sinks: RoPE tables need %d bytes of shared memory (max %d)", tab,
              kTableMaxBytes);
    return PRSINK_ERR_UNSUPPORTED;
  }
  const int smem = kRotGroups * 2 * Layout<D>::kTileBytes + tab + 1024;
  static int allowed[64] = {0};
  rc = allow_smem(prsink_rotate_kernel<D, RT, RH>, smem, allowed, "prsink_rotate_sinks");
  if (rc) return rc;
  int n_sm = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  // work items: the (head, key tile) pairs of the rotated slots; one CTA per SM, kRotGroups
  // pipelines each, stream them
  const long long items = static_cast<long long>(H) * ((g.T + BN - 1) / BN);
  const long long ctas = (items + kRotGroups - 1) / kRotGroups;
  const int grid = static_cast<int>(ctas < n_sm ? ctas : n_sm);
  prsink_rotate_kernel<D, RT, RH><<<grid, kRotThreads, smem, st>>>(ms, md, p);
  count_launch();
  return check_launch("prsink_rotate_sinks");
}

// Split of the last wave.  Units (head, pair of query tiles) run one CTA per SM; when the
// last wave holds r < #SM units, each of those runs as S = min(#SM / r, kMaxSplit) CTAs over
// equal shares of the key tiles, so the last wave takes ~1/S of a unit's time.
struct SplitPlan {
  int split_base, n_split, r;
  size_t o_bytes, ml_bytes, cnt_bytes;       // scratch regions, each 256-byte aligned
  size_t total() const { return o_bytes + ml_bytes + cnt_bytes; }
};

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static SplitPlan plan_split(const Geometry& g, int H, int D) {
  SplitPlan sp{};
  const int nqb = static_cast<int>((g.L_blk + NQ * BM - 1) / (NQ * BM));
  const int units = nqb * H;
  int n_sm = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  sp.split_base = units;
  sp.n_split = 1;
  if (units <= 0 || n_sm <= 0) return sp;
  const int waves = (units + n_sm - 1) / n_sm;
  const int r = units - (waves - 1) * n_sm;
  int S = n_sm / r;
  if (S > kMaxSplit) S = kMaxSplit;
  const int tiles = static_cast<int>((g.T + BN - 1) / BN);
  if (S > tiles) S = tiles;
  if (S < 2) return sp;
  sp.split_base = units - r;
  sp.n_split = S;
  sp.r = r;
  const size_t parts = static_cast<size_t>(r) * S * (NQ * BM);
  sp.o_bytes = align256(parts * D * sizeof(float));
  sp.ml_bytes = align256(parts * sizeof(float2));
  sp.cnt_bytes = align256(static_cast<size_t>(r) * sizeof(int));
  return sp;
}

// Self-test of the attention kernel's abort path (per host thread, one call).
static thread_local long long g_debug_stall_ns = 0;

// Parameters shared by every kernel of this file, from the layout (validated by the caller).
static int fill_params(const prsink_layout* layout, const Geometry& g, Params& p,
                       const char* what) {
  const int D = layout->head_dim;
  p = Params{};
  p.H = layout->n_heads;
  p.L_blk = static_cast<int>(g.L_blk);
  p.T = static_cast<int>(g.T);
  p.L_f = static_cast<int>(g.L_f);
  p.grid_h = layout->grid_h;
  p.grid_w = layout->grid_w;
  p.n_slots = g.n_slots;
  for (int s = 0; s <= g.n_slots; ++s) p.slot_start[s] = static_cast<int>(g.slot_start[s]);
  const int R = layout->ring_slots;
  const int Bf = layout->frames_per_block;
  const long long b = layout->block_index;
  p.slot_frame[PRSINK_SLOT_REF] = 0;
  p.slot_frame[PRSINK_SLOT_STATIC] = layout->ref_frames;
  p.slot_frame[PRSINK_SLOT_DYNAMIC] = layout->ref_frames + Bf;
  for (int s = 0; s < R; ++s) {
    // ring slot s holds block b' = s (mod R), b' in [b-R+1, b]; its age rank is b'-(b-R+1)
    const long long oldest = b - R + 1;
    const int rank = static_cast<int>((((s - oldest) % R) + R) % R);
    p.slot_frame[PRSINK_SLOT_RING0 + s] = layout->ref_frames + (2 + rank) * Bf;
  }
  p.q_frame = layout->ref_frames + (2 + R - 1) * Bf;
  p.n_frames = layout->ref_frames + (2 + R) * Bf;
  p.valid_mask = layout->valid_mask & ((1u << g.n_slots) - 1u);
  p.rope_mode = layout->rope_mode;
  if (p.rope_mode == 3) {
    p.rd[0] = layout->rope_split[0] / 2;
    p.rd[1] = layout->rope_split[1] / 2;
    p.rd[2] = layout->rope_split[2] / 2;
    p.tab_h_off = p.n_frames * p.rd[0];
    p.tab_w_off = p.tab_h_off + layout->grid_h * p.rd[1];
    p.tab_entries = p.tab_w_off + layout->grid_w * p.rd[2];
  } else {
    p.rd[0] = D / 2;
    p.rd[1] = 0;
    p.rd[2] = 0;
    p.tab_h_off = p.n_frames * (D / 2);
    p.tab_w_off = p.tab_h_off + p.L_f * (D / 2);
    p.tab_entries = p.tab_w_off;
  }
  p.step_y = BN / layout->grid_w;
  p.step_x = BN % layout->grid_w;
  if ((g.T + BN - 1) / BN > kMaxTiles) {
    set_error("%s: %lld keys exceed the %d-tile limit", what, g.T, kMaxTiles);
    return PRSINK_ERR_UNSUPPORTED;
  }
  if (p.tab_entries * 8 > kTableMaxBytes) {
    set_error("%s: RoPE tables need %d bytes of shared memory (max %d)", what,
              p.tab_entries * 8, kTableMaxBytes);
    return PRSINK_ERR_UNSUPPORTED;
  }
  p.log2_base = std::log2(static_cast<double>(layout->rope_base));
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.status = status_word_ptr();
  p.timeout_ns = 2000000000ull;
  p.cur_slot = -1;
  p.nqb = static_cast<int>((g.L_blk + NQ * BM - 1) / (NQ * BM));
  p.split_base = p.nqb * layout->n_heads;     // no split unless a caller plans one
  p.n_split = 1;
  if (g_debug_stall_ns > 0) {           // armed by prsink_debug_attention_stall: one call only
    p.debug_stall = 1;
    p.timeout_ns = static_cast<unsigned long long>(g_debug_stall_ns);
    g_debug_stall_ns = 0;
  }
  if (!p.status) return PRSINK_ERR_LAUNCH;
  return PRSINK_OK;
}

static bool grouped_split(const prsink_layout* L, const Params& p) {
  return L->head_dim == 128 && p.rope_mode == 3 && p.rd[0] == 22 && p.rd[1] == 21;
}

template <bool kFused>
static int dispatch(const prsink_layout* L, const Geometry& g, const Buffers& b, Params& p,
                    cudaStream_t st) {
  if (grouped_split(L, p)) return launch<128, 22, 21, kFused>(L, g, b, p, st);   // 44/42/42
  return L->head_dim == 128 ? launch<128, 0, 0, kFused>(L, g, b, p, st)
                            : launch<64, 0, 0, kFused>(L, g, b, p, st);
}

// Common checks of the attention entry points.
static int check_attention_args(const prsink_layout* layout, Geometry* g, const char* what,
                                std::initializer_list<const void*> bufs, const float* lse) {
  int rc = geometry(layout, g);
  if (rc) return rc;
  for (const void* ptr : bufs)
    if (!ptr) {
      set_error("%s: null pointer", what);
      return PRSINK_ERR_ARG;
    }
  const int D = layout->head_dim;
  if (D != 64 && D != 128) {
    set_error("%s: head_dim %d not supported (64 or 128)", what, D);
    return PRSINK_ERR_UNSUPPORTED;
  }
  for (const void* ptr : bufs)
    if (!aligned16(ptr)) {
      set_error("%s: every K/V/Q/out buffer must be 16-byte aligned", what);
      return PRSINK_ERR_ALIGN;
    }
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) {
    set_error("%s: lse must be 4-byte aligned", what);
    return PRSINK_ERR_ALIGN;
  }
  return PRSINK_OK;
}

}  // namespace attn
}  // namespace prsink

using namespace prsink;

extern "C" int prsink_attention(const prsink_layout* layout, const void* q, const void* k_cache,
                                const void* v_cache, void* out, float* lse,
                                const long long* dyn_src, void* stream) {
  using namespace prsink::attn;
  Geometry g;
  int rc = check_attention_args(layout, &g, "prsink_attention", {q, k_cache, v_cache, out}, lse);
  if (rc) return rc;
  Params p;
  rc = fill_params(layout, g, p, "prsink_attention");
  if (rc) return rc;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dyn_src = dyn_src;
  if (g.L_blk == 0) return PRSINK_OK;
  const Buffers b{q, k_cache, v_cache, nullptr, nullptr, nullptr, nullptr};
  return dispatch<false>(layout, g, b, p, static_cast<cudaStream_t>(stream));
}

extern "C" long long prsink_attention_scratch_bytes(const prsink_layout* layout) {
  using namespace prsink::attn;
  Geometry g;
  if (geometry(layout, &g)) return -1;
  return static_cast<long long>(plan_split(g, layout->n_heads, layout->head_dim).total());
}

// Shared by the split entry points: plan, carve `scratch` and launch.
static int attention_split_impl(const char* what, const prsink_layout* layout, const void* q,
                                const void* k_cache, const void* v_cache, void* out, float* lse,
                                const long long* dyn_src, void* scratch,
                                long long scratch_bytes, void* stream) {
  using namespace prsink::attn;
  Geometry g;
  int rc = check_attention_args(layout, &g, what, {q, k_cache, v_cache, out}, lse);
  if (rc) return rc;
  Params p;
  rc = fill_params(layout, g, p, what);
  if (rc) return rc;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dyn_src = dyn_src;
  if (g.L_blk == 0) return PRSINK_OK;
  const SplitPlan sp = plan_split(g, layout->n_heads, layout->head_dim);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sp.n_split > 1) {
    if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u) ||
        scratch_bytes < static_cast<long long>(sp.total())) {
      set_error("%s: scratch must be 256-byte aligned and hold %zu bytes (got %lld)", what,
                sp.total(), scratch_bytes);
      return PRSINK_ERR_ARG;
    }
    char* base = static_cast<char*>(scratch);
    p.part_o = reinterpret_cast<float*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + sp.o_bytes);
    p.part_cnt = reinterpret_cast<int*>(base + sp.o_bytes + sp.ml_bytes);
    p.split_base = sp.split_base;
    p.n_split = sp.n_split;
    // the arrival counters start at zero (the combining CTA also resets them)
    if (cudaMemsetAsync(p.part_cnt, 0, sp.cnt_bytes, st) != cudaSuccess)
      return check_launch(what);
  }
  const Buffers b{q, k_cache, v_cache, nullptr, nullptr, nullptr, nullptr};
  return dispatch<false>(layout, g, b, p, st);
}

extern "C" int prsink_attention_split(const prsink_layout* layout, const void* q,
                                      const void* k_cache, const void* v_cache, void* out,
                                      float* lse, const long long* dyn_src, void* scratch,
                                      long long scratch_bytes, void* stream) {
  return attention_split_impl("prsink_attention_split", layout, q, k_cache, v_cache, out, lse,
                              dyn_src, scratch, scratch_bytes, stream);
}

// ---- allocation-free form of prsink_attention_split ------------------------------------
// For callers that cannot allocate device memory: an embedding runtime that owns the device's
// memory pool and forbids allocations outside it (a framework allocator, a memory-capped
// serving process), or a real-time loop that may not call the allocator (cudaMalloc can
// synchronise the device and take milliseconds).  Their scratch is this file-scope device
// array, so the library allocates nothing when it is used; every GPU that loads the library
// holds it from module load until the process exits.
// 20 MiB: a split plan has at most one partial per SM (r units x S shares <= #SM); on a
// 148-SM device with head_dim 128 that is 148 x 256 rows x (512 + 8) B + counters = 19.7 MB.
constexpr size_t kStaticSplitScratchBytes = 20ull << 20;
static __device__ __align__(256) unsigned char g_split_scratch[kStaticSplitScratchBytes];

// Device address of g_split_scratch on the current device.  In host code the symbol's name is
// only a host-side stand-in, not a device address, so the address is looked up once per device
// (with that device current) and kept.
static void* static_split_scratch(const char* what) {
  static void* addr[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    set_error("%s: no current CUDA device", what);
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_split_scratch);
    if (e != cudaSuccess || !ptr) {
      set_error("%s: cudaGetSymbolAddress of the scratch array failed: %s", what,
                cudaGetErrorString(e));
      return nullptr;
    }
    addr[dev] = ptr;
  }
  return addr[dev];
}

extern "C" int prsink_attention_split_noalloc(const prsink_layout* layout, const void* q,
                                              const void* k_cache, const void* v_cache,
                                              void* out, float* lse, const long long* dyn_src,
                                              void* stream) {
  using namespace prsink::attn;
  const char* what = "prsink_attention_split_noalloc";
  Geometry g;
  int rc = geometry(layout, &g);
  if (rc) return rc;
  const size_t need = plan_split(g, layout->n_heads, layout->head_dim).total();
  if (need > kStaticSplitScratchBytes) {
    set_error("%s: this layout needs %zu bytes of split scratch, more than the %zu-byte "
              "static array; use prsink_attention_split with caller scratch", what, need,
              kStaticSplitScratchBytes);
    return PRSINK_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  if (need) {
    scratch = static_split_scratch(what);
    if (!scratch) return PRSINK_ERR_LAUNCH;
  }
  return attention_split_impl(what, layout, q, k_cache, v_cache, out, lse, dyn_src, scratch,
                              static_cast<long long>(kStaticSplitScratchBytes), stream);
}

// Shared by the fused entry points; `scratch` may be null (no split).
static int attention_fused_impl(const char* what, const prsink_layout* layout, const void* q,
                                const void* k_new, const void* v_new, const void* k_rot,
                                void* k_cache, void* v_cache, void* out, float* lse,
                                const long long* dyn_src, void* scratch, long long scratch_bytes,
                                bool split, void* stream) {
  using namespace prsink::attn;
  Geometry g;
  int rc = check_attention_args(layout, &g, what, {q, k_new, v_new, k_rot, k_cache, v_cache, out},
                                lse);
  if (rc) return rc;
  if (k_rot == k_cache) {
    set_error("%s: k_rot must be a buffer of its own", what);
    return PRSINK_ERR_ARG;
  }
  Params p;
  rc = fill_params(layout, g, p, what);
  if (rc) return rc;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dyn_src = dyn_src;
  p.cur_slot = PRSINK_SLOT_RING0 + static_cast<int>(layout->block_index % layout->ring_slots);
  p.n_cur_tiles = static_cast<int>((g.L_blk + BN - 1) / BN);
  if ((g.T + BN - 1) / BN + p.n_cur_tiles > kMaxTiles) {
    set_error("%s: %lld keys exceed the tile limit", what, g.T);
    return PRSINK_ERR_UNSUPPORTED;
  }
  if (g.L_blk == 0) return PRSINK_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (split) {
    // a tile of the current block is stored by whichever share of its unit holds it
    const SplitPlan sp = plan_split(g, layout->n_heads, layout->head_dim);
    if (sp.n_split > 1) {
      if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u) ||
          scratch_bytes < static_cast<long long>(sp.total())) {
        set_error("%s: scratch must be 256-byte aligned and hold %zu bytes (got %lld)", what,
                  sp.total(), scratch_bytes);
        return PRSINK_ERR_ARG;
      }
      char* base = static_cast<char*>(scratch);
      p.part_o = reinterpret_cast<float*>(base);
      p.part_ml = reinterpret_cast<float2*>(base + sp.o_bytes);
      p.part_cnt = reinterpret_cast<int*>(base + sp.o_bytes + sp.ml_bytes);
      p.split_base = sp.split_base;
      p.n_split = sp.n_split;
      if (cudaMemsetAsync(p.part_cnt, 0, sp.cnt_bytes, st) != cudaSuccess)
        return check_launch(what);
    }
  }
  const Buffers b{q, k_rot, v_cache, k_new, v_new, k_cache, v_cache};
  return dispatch<true>(layout, g, b, p, st);
}

extern "C" int prsink_attention_fused(const prsink_layout* layout, const void* q,
                                      const void* k_new, const void* v_new, const void* k_rot,
                                      void* k_cache, void* v_cache, void* out, float* lse,
                                      const long long* dyn_src, void* stream) {
  return attention_fused_impl("prsink_attention_fused", layout, q, k_new, v_new, k_rot, k_cache,
                              v_cache, out, lse, dyn_src, nullptr, 0, false, stream);
}

extern "C" int prsink_attention_fused_split(const prsink_layout* layout, const void* q,
                                            const void* k_new, const void* v_new,
                                            const void* k_rot, void* k_cache, void* v_cache,
                                            void* out, float* lse, const long long* dyn_src,
                                            void* scratch, long long scratch_bytes,
                                            void* stream) {
  return attention_fused_impl("prsink_attention_fused_split", layout, q, k_new, v_new, k_rot,
                              k_cache, v_cache, out, lse, dyn_src, scratch, scratch_bytes, true,
                              stream);
}

extern "C" int prsink_rotate_sinks(const prsink_layout* layout, const void* k_cache,
                                   void* k_rot, unsigned slot_mask, const int* dyn_flag,
                                   const long long* dyn_src, void* stream) {
  using namespace prsink::attn;
  Geometry g;
  int rc = check_attention_args(layout, &g, "prsink_rotate_sinks", {k_cache, k_rot}, nullptr);
  if (rc) return rc;
  if (k_rot == k_cache) {
    set_error("prsink_rotate_sinks: k_rot must be a buffer of its own");
    return PRSINK_ERR_ARG;
  }
  Params p;
  rc = fill_params(layout, g, p, "prsink_rotate_sinks");
  if (rc) return rc;
  p.cur_slot = PRSINK_SLOT_RING0 + static_cast<int>(layout->block_index % layout->ring_slots);
  p.rot_mask = slot_mask;
  p.rot_dyn_flag = dyn_flag;
  p.dyn_src = dyn_src;
  if ((slot_mask & p.valid_mask & ~(1u << p.cur_slot)) == 0) return PRSINK_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (grouped_split(layout, p)) return launch_rotate<128, 22, 21>(layout, g, k_cache, k_rot, p, st);
  return layout->head_dim == 128 ? launch_rotate<128, 0, 0>(layout, g, k_cache, k_rot, p, st)
                                 : launch_rotate<64, 0, 0>(layout, g, k_cache, k_rot, p, st);
}

extern "C" int prsink_debug_attention_stall(long long timeout_ns) {
  if (timeout_ns < 10000) timeout_ns = 10000;
  if (timeout_ns > 1000000000ll) timeout_ns = 1000000000ll;
  prsink::attn::g_debug_stall_ns = timeout_ns;
  return PRSINK_OK;
}
