// Pose side of the PR-Sink step: the 558-d fingerprint, retrieval r(b) = argmax phi_b.phi_i
// (excluding block b-1) with the dynamic-sink fill, and the diversity-driven bank update with
// the bank store.  The arithmetic is a few thousand multiply-adds: each decision is one CTA
// (one warp per dot product, warp-shuffle reductions in float64), followed by an HBM-bound
// predicated copy kernel that reads the decision from device memory, so no host sync is
// needed between the decision and the copy.
#include <cmath>

#include "prsink_internal.cuh"

namespace prsink {

int launch_bank_cache_copy(const prsink_layout* L, const Geometry& g, int M, int n_layers,
                           const void* bank_kv, const void* cache_kv, bool to_cache, int slot,
                           const int* sel, const int* flag, int want, cudaStream_t st,
                           float blend_alpha);

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Dot product of two 558-vectors by one warp, float64 accumulation.
__device__ __forceinline__ double warp_dot(const float* __restrict__ a,
                                           const float* __restrict__ b, int lane) {
  double s = 0.0;
  for (int i = lane; i < PRSINK_FP_DIM; i += 32) s += static_cast<double>(a[i]) * b[i];
  return warp_sum(s);
}

// ---------------------------------------------------------------------------- fingerprint
__global__ void __launch_bounds__(256)
fingerprint_kernel(const float* __restrict__ kp, const unsigned char* __restrict__ ok,
                   float* __restrict__ phi) {
  __shared__ double part[8];
  __shared__ float v[PRSINK_FP_DIM];
  constexpr int per = PRSINK_FP_KEYPOINTS * PRSINK_FP_CHANNELS;
  double s = 0.0;
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x) {
    const float x = ok[i / per] ? kp[i] : 0.f;      // failed frame -> zeros
    v[i] = x;
    s += static_cast<double>(x) * x;
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  double n2 = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) n2 += part[w];
  const double inv = n2 > 0.0 ? 1.0 / sqrt(n2) : 0.0;
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x)
    phi[i] = static_cast<float>(static_cast<double>(v[i]) * inv);
}

// ---------------------------------------------------------------------------- retrieval
// One warp per bank entry computes phi_b . phi_i; warp 0 then takes the argmax over eligible
// entries with a shuffle reduction (ties -> lowest slot).  With `frame_ok` given, a block with
// fewer than `min_detected` detected frames retrieves nothing (fallback to Static Sink +
// window: the dynamic sink stays empty for the block).
__global__ void __launch_bounds__(1024)
retrieve_kernel(const float* __restrict__ phi_b, const float* __restrict__ bank_phi,
                const long long* __restrict__ bank_src, const int* __restrict__ bank_count,
                int M, long long exclude, int* __restrict__ r_out, float* __restrict__ score_out,
                int* __restrict__ copy_out, long long* __restrict__ dyn_src,
                const unsigned char* __restrict__ frame_ok, int min_detected) {
  __shared__ double score[PRSINK_MAX_BANK];
  __shared__ float q[PRSINK_FP_DIM];
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x) q[i] = phi_b[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int count = *bank_count;
  if (frame_ok) {
    int detected = 0;
    for (int f = 0; f < PRSINK_FP_FRAMES; ++f) detected += frame_ok[f] ? 1 : 0;
    if (detected < min_detected) count = 0;        // nothing is eligible
  }
  if (warp < M && warp < count) {
    const double d = warp_dot(q, bank_phi + static_cast<size_t>(warp) * PRSINK_FP_DIM, lane);
    if (lane == 0) score[warp] = d;
  }
  __syncthreads();
  if (warp != 0) return;
  const bool elig = lane < M && lane < count && bank_src[lane] != exclude;
  double best = elig ? score[lane] : -INFINITY;
  int idx = elig ? lane : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (ob > best || (ob == best && oi < idx)) { best = ob; idx = oi; }
  }
  if (lane == 0) {
    const int r = idx == 0x7fffffff ? -1 : idx;
    const long long old = *dyn_src;
    const long long src = r >= 0 ? bank_src[r] : -1;
    *r_out = r;
    if (score_out) *score_out = r >= 0 ? static_cast<float>(best) : -INFINITY;
    *copy_out = (r >= 0 && src != old) ? 1 : 0;
    *dyn_src = src;
  }
}

// ---------------------------------------------------------------------------- bank update
// Policies (variants of the pages' frozen bank, digest weaknesses 3 and 5).
constexpr int kBankFrozen = 0, kBankDecay = 1, kBankGated = 2;
constexpr int kModeNone = 0, kModeStore = 1, kModeBlend = 2;

struct BankPolicy {
  int kind;            // kBankFrozen / kBankDecay / kBankGated
  int write_blocks;    // the diversity rule runs for b < write_blocks
  float alpha;         // decay: weight of the block in the moving average
  float gate;          // gated: refresh when min_i ||phi_b - phi_i|| > gate
};

__device__ __forceinline__ double warp_dist2(const float* __restrict__ a,
                                             const float* __restrict__ b, int lane) {
  double s = 0.0;
  for (int i = lane; i < PRSINK_FP_DIM; i += 32) {
    const double t = static_cast<double>(a[i]) - static_cast<double>(b[i]);
    s += t * t;
  }
  return warp_sum(s);
}

// Diversity rule: options keep (index 0) or replace slot j (index 1+j).  With G the Gram
// matrix of the bank and c_i = phi_i . phi_b, the pair sum of "replace j" is
//   S_keep - sum_{i != j} G_ij + sum_{i != j} c_i,
// and every option has the same pair count, so the least pair sum is the least mean.
// After the freeze (b >= write_blocks) the frozen policy writes nothing; the gated policy runs
// the diversity rule for a block farther than the gate from every entry; the decay policy
// averages the block into its nearest entry (argmax c_i): phi_j <- normalise((1 - alpha) phi_j
// + alpha phi_b) in float64, and the K/V blend is launched on the mode word.
__global__ void __launch_bounds__(1024)
bank_update_kernel(float* __restrict__ bank_phi, long long* __restrict__ bank_src,
                   int* __restrict__ bank_count, int M, const float* __restrict__ phi_b,
                   long long b, BankPolicy pol, int* __restrict__ action_out,
                   int* __restrict__ mode_out) {
  __shared__ double G[PRSINK_MAX_BANK][PRSINK_MAX_BANK + 1];   // row j: G[j][i]; col M: c_j
  __shared__ double D2[PRSINK_MAX_BANK];                        // ||phi_i - phi_b||^2
  __shared__ double part[32];
  __shared__ float q[PRSINK_FP_DIM];
  __shared__ int action_s, mode_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int count = *bank_count;
  const int used = count < M ? count : M;
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x) q[i] = phi_b[i];
  if (threadIdx.x == 0) { action_s = -1; mode_s = kModeNone; }
  __syncthreads();
  const bool frozen_phase = b >= pol.write_blocks;
  const bool may_diversify = !frozen_phase || pol.kind == kBankGated;
  // similarities to the candidate (and distances for the gate) of every entry in use
  for (int i = warp; i < used; i += nw) {
    const float* a = bank_phi + static_cast<size_t>(i) * PRSINK_FP_DIM;
    const double c = warp_dot(a, q, lane);
    double d2 = 0.0;
    if (pol.kind == kBankGated && frozen_phase) d2 = warp_dist2(a, q, lane);
    if (lane == 0) { G[i][M] = c; D2[i] = d2; }
  }
  if (may_diversify && count >= M) {
    // pairs (i, j) with i < j of the full bank
    const int n_pairs = M * (M - 1) / 2;
    for (int p = warp; p < n_pairs; p += nw) {
      int i = 0, rem = p;                          // unrank p into i < j
      while (rem >= M - 1 - i) { rem -= M - 1 - i; ++i; }
      const int j = i + 1 + rem;
      const double d = warp_dot(bank_phi + static_cast<size_t>(i) * PRSINK_FP_DIM,
                                bank_phi + static_cast<size_t>(j) * PRSINK_FP_DIM, lane);
      if (lane == 0) { G[i][j] = d; G[j][i] = d; }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int action = -1, mode = kModeNone;
    bool diversify = !frozen_phase;
    if (frozen_phase && pol.kind == kBankGated) {
      double dmin = INFINITY;
      for (int i = 0; i < used; ++i) dmin = fmin(dmin, D2[i]);
      diversify = used == 0 || sqrt(dmin) > static_cast<double>(pol.gate);
    }
    if (diversify) {
      if (count < M) {
        action = count;
      } else {
        double keep = 0.0;
        for (int i = 0; i < M; ++i)
          for (int j = i + 1; j < M; ++j) keep += G[i][j];
        double best = keep;
        for (int j = 0; j < M; ++j) {
          double s = keep;
          for (int i = 0; i < M; ++i)
            if (i != j) s += G[i][M] - G[i][j];
          if (s < best) { best = s; action = j; }
        }
      }
      if (action >= 0) mode = kModeStore;
    } else if (frozen_phase && pol.kind == kBankDecay && pol.alpha > 0.f && used > 0) {
      int jb = 0;
      for (int i = 1; i < used; ++i)
        if (G[i][M] > G[jb][M]) jb = i;            // ties -> lowest slot
      action = jb;
      mode = kModeBlend;
    }
    action_s = action;
    mode_s = mode;
    *action_out = action;
    if (mode_out) *mode_out = mode;
    if (action >= 0) {
      bank_src[action] = b;
      if (mode == kModeStore && count < M) *bank_count = count + 1;
    }
  }
  __syncthreads();
  const int a = action_s;
  if (mode_s == kModeStore) {
    for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x)
      bank_phi[static_cast<size_t>(a) * PRSINK_FP_DIM + i] = q[i];
  } else if (mode_s == kModeBlend) {
    float* e = bank_phi + static_cast<size_t>(a) * PRSINK_FP_DIM;
    const double w_new = static_cast<double>(pol.alpha);
    const double w_old = static_cast<double>(1.0f - pol.alpha);   // the float32 weight
    // one element per thread (the kernel runs with 1024 >= 558 threads)
    const int i = threadIdx.x;
    const double t = i < PRSINK_FP_DIM
                         ? w_old * static_cast<double>(e[i]) + w_new * static_cast<double>(q[i])
                         : 0.0;
    double s = warp_sum(t * t);
    if (lane == 0) part[warp] = s;
    __syncthreads();
    double n2 = 0.0;
    for (int w = 0; w < nw; ++w) n2 += part[w];
    const double inv = n2 > 0.0 ? 1.0 / sqrt(n2) : 1.0;
    if (i < PRSINK_FP_DIM) e[i] = static_cast<float>(t * inv);
  }
}

static bool bad_bank(int M) { return M < 1 || M > PRSINK_MAX_BANK; }

}  // namespace prsink

using namespace prsink;

extern "C" int prsink_fingerprint(const float* kp, const unsigned char* frame_ok, float* phi,
                                  void* stream) {
  if (!kp || !frame_ok || !phi) {
    set_error("prsink_fingerprint: null pointer");
    return PRSINK_ERR_ARG;
  }
  fingerprint_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(kp, frame_ok, phi);
  count_launch();
  return check_launch("prsink_fingerprint");
}

// Validates the optional K/V copy arguments shared by retrieval and the bank update.
static int copy_args(const char* fn, const prsink_layout* layout, const void* bank_kv,
                     const void* cache_kv, int n_layers, Geometry* g, bool* do_copy) {
  *do_copy = bank_kv || cache_kv || n_layers;
  if (!*do_copy) return PRSINK_OK;
  int rc = geometry(layout, g);
  if (rc) return rc;
  if (!bank_kv || !cache_kv || n_layers < 1) {
    set_error("%s: bank_kv, cache_kv and n_layers >= 1 go together", fn);
    return PRSINK_ERR_ARG;
  }
  if (!aligned16(bank_kv) || !aligned16(cache_kv) || (layout->head_dim * 2) % 16) {
    set_error("%s: K/V buffers must be 16-byte aligned", fn);
    return PRSINK_ERR_ALIGN;
  }
  return PRSINK_OK;
}

static int retrieve_impl(const char* fn, const prsink_layout* layout, const float* phi_b,
                         const unsigned char* frame_ok, int min_detected, const float* bank_phi,
                         const long long* bank_src, const int* bank_count, int M,
                         long long exclude_block, int* r_out, float* score_out, int* copy_out,
                         long long* dyn_src, const void* bank_kv, void* cache_kv, int n_layers,
                         void* stream) {
  if (!phi_b || !bank_phi || !bank_src || !bank_count || !r_out || !copy_out || !dyn_src) {
    set_error("%s: null pointer", fn);
    return PRSINK_ERR_ARG;
  }
  if (bad_bank(M)) {
    set_error("%s: M = %d outside [1, %d]", fn, M, PRSINK_MAX_BANK);
    return PRSINK_ERR_ARG;
  }
  Geometry g{};
  bool do_copy = false;
  int rc = copy_args(fn, layout, bank_kv, cache_kv, n_layers, &g, &do_copy);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  retrieve_kernel<<<1, 32 * M, 0, st>>>(phi_b, bank_phi, bank_src, bank_count, M, exclude_block,
                                        r_out, score_out, copy_out, dyn_src, frame_ok,
                                        min_detected);
  count_launch();
  rc = check_launch(fn);
  if (rc || !do_copy) return rc;
  return launch_bank_cache_copy(layout, g, M, n_layers, bank_kv, cache_kv, /*to_cache=*/true,
                                PRSINK_SLOT_DYNAMIC, r_out, copy_out, 1, st, -1.f);
}

static int bank_update_impl(const char* fn, const prsink_layout* layout, const BankPolicy& pol,
                            float* bank_phi, long long* bank_src, int* bank_count, int M,
                            const float* phi_b, long long b, int* action_out, int* mode_out,
                            const void* cache_kv, void* bank_kv, int n_layers, void* stream) {
  if (!bank_phi || !bank_src || !bank_count || !phi_b || !action_out) {
    set_error("%s: null pointer", fn);
    return PRSINK_ERR_ARG;
  }
  if (bad_bank(M) || b < 0) {
    set_error("%s: M = %d outside [1, %d] or b = %lld < 0", fn, M, PRSINK_MAX_BANK, b);
    return PRSINK_ERR_ARG;
  }
  Geometry g{};
  bool do_copy = false;
  int rc = copy_args(fn, layout, bank_kv, cache_kv, n_layers, &g, &do_copy);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  static_assert(PRSINK_FP_DIM <= 1024, "the blend takes one fingerprint element per thread");
  bank_update_kernel<<<1, 1024, 0, st>>>(bank_phi, bank_src, bank_count, M, phi_b, b, pol,
                                         action_out, mode_out);
  count_launch();
  rc = check_launch(fn);
  if (rc || !do_copy) return rc;
  const int ring = PRSINK_SLOT_RING0 + static_cast<int>(b % layout->ring_slots);
  // store: the block's clean K/V replaces the entry (predicated on the action, and on the
  // mode word when there is one); decayed write: the entry is averaged with the block
  rc = launch_bank_cache_copy(layout, g, M, n_layers, bank_kv, cache_kv, /*to_cache=*/false,
                              ring, action_out, mode_out, kModeStore, st, -1.f);
  if (rc || pol.kind != kBankDecay) return rc;
  return launch_bank_cache_copy(layout, g, M, n_layers, bank_kv, cache_kv, /*to_cache=*/false,
                                ring, action_out, mode_out, kModeBlend, st, pol.alpha);
}

extern "C" int prsink_retrieve(const prsink_layout* layout, const float* phi_b,
                               const float* bank_phi, const long long* bank_src,
                               const int* bank_count, int M, long long exclude_block,
                               int* r_out, float* score_out, int* copy_out, long long* dyn_src,
                               const void* bank_kv, void* cache_kv, int n_layers, void* stream) {
  return retrieve_impl("prsink_retrieve", layout, phi_b, nullptr, 0, bank_phi, bank_src,
                       bank_count, M, exclude_block, r_out, score_out, copy_out, dyn_src,
                       bank_kv, cache_kv, n_layers, stream);
}

extern "C" int prsink_retrieve_fallback(const prsink_layout* layout, const float* phi_b,
                                        const unsigned char* frame_ok, int min_detected,
                                        const float* bank_phi, const long long* bank_src,
                                        const int* bank_count, int M, long long exclude_block,
                                        int* r_out, float* score_out, int* copy_out,
                                        long long* dyn_src, const void* bank_kv, void* cache_kv,
                                        int n_layers, void* stream) {
  if (!frame_ok || min_detected < 0 || min_detected > PRSINK_FP_FRAMES) {
    set_error("prsink_retrieve_fallback: frame_ok must be given and min_detected in [0, %d]",
              PRSINK_FP_FRAMES);
    return PRSINK_ERR_ARG;
  }
  return retrieve_impl("prsink_retrieve_fallback", layout, phi_b, frame_ok, min_detected,
                       bank_phi, bank_src, bank_count, M, exclude_block, r_out, score_out,
                       copy_out, dyn_src, bank_kv, cache_kv, n_layers, stream);
}

extern "C" int prsink_bank_update(const prsink_layout* layout, float* bank_phi,
                                  long long* bank_src, int* bank_count, int M,
                                  const float* phi_b, long long b, int write_blocks,
                                  int* action_out, const void* cache_kv, void* bank_kv,
                                  int n_layers, void* stream) {
  const BankPolicy pol{kBankFrozen, write_blocks, 0.f, 0.f};
  return bank_update_impl("prsink_bank_update", layout, pol, bank_phi, bank_src, bank_count, M,
                          phi_b, b, action_out, nullptr, cache_kv, bank_kv, n_layers, stream);
}

extern "C" int prsink_bank_update_policy(const prsink_layout* layout,
                                         const prsink_bank_policy* policy, float* bank_phi,
                                         long long* bank_src, int* bank_count, int M,
                                         const float* phi_b, long long b, int* action_out,
                                         int* mode_out, const void* cache_kv, void* bank_kv,
                                         int n_layers, void* stream) {
  if (!policy || !mode_out) {
    set_error("prsink_bank_update_policy: policy and mode_out must be given");
    return PRSINK_ERR_ARG;
  }
  const int k = policy->kind;
  if ((k != PRSINK_BANK_FROZEN && k != PRSINK_BANK_DECAY && k != PRSINK_BANK_GATED) ||
      policy->write_blocks < 0 || !(policy->alpha >= 0.f && policy->alpha <= 1.f) ||
      !std::isfinite(policy->gate)) {
    set_error("prsink_bank_update_policy: invalid policy (kind %d, write_blocks %d, alpha %g, "
              "gate %g)", k, policy->write_blocks, policy->alpha, policy->gate);
    return PRSINK_ERR_ARG;
  }
  static_assert(PRSINK_BANK_FROZEN == kBankFrozen && PRSINK_BANK_DECAY == kBankDecay &&
                PRSINK_BANK_GATED == kBankGated, "policy kinds");
  static_assert(PRSINK_BANK_MODE_STORE == kModeStore && PRSINK_BANK_MODE_BLEND == kModeBlend,
                "mode words");
  const BankPolicy pol{k, policy->write_blocks, policy->alpha, policy->gate};
  return bank_update_impl("prsink_bank_update_policy", layout, pol, bank_phi, bank_src,
                          bank_count, M, phi_b, b, action_out, mode_out, cache_kv, bank_kv,
                          n_layers, stream);
}
