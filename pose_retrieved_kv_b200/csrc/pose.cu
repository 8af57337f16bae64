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
                           const int* sel, const int* flag, cudaStream_t st);

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
// entries with a shuffle reduction (ties -> lowest slot).
__global__ void __launch_bounds__(1024)
retrieve_kernel(const float* __restrict__ phi_b, const float* __restrict__ bank_phi,
                const long long* __restrict__ bank_src, const int* __restrict__ bank_count,
                int M, long long exclude, int* __restrict__ r_out, float* __restrict__ score_out,
                int* __restrict__ copy_out, long long* __restrict__ dyn_src) {
  __shared__ double score[PRSINK_MAX_BANK];
  __shared__ float q[PRSINK_FP_DIM];
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x) q[i] = phi_b[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int count = *bank_count;
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
// Options: keep (index 0) or replace slot j (index 1+j).  With G the Gram matrix of the bank
// and c_i = phi_i . phi_b, the pair sum of "replace j" is
//   S_keep - sum_{i != j} G_ij + sum_{i != j} c_i,
// and every option has the same pair count, so the least pair sum is the least mean.
__global__ void __launch_bounds__(1024)
bank_update_kernel(float* __restrict__ bank_phi, long long* __restrict__ bank_src,
                   int* __restrict__ bank_count, int M, const float* __restrict__ phi_b,
                   long long b, int write_blocks, int* __restrict__ action_out) {
  __shared__ double G[PRSINK_MAX_BANK][PRSINK_MAX_BANK + 1];   // row j: G[j][i]; col M: c_j
  __shared__ float q[PRSINK_FP_DIM];
  __shared__ int action_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int count = *bank_count;
  for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x) q[i] = phi_b[i];
  if (threadIdx.x == 0) action_s = -1;
  __syncthreads();
  const bool decide = b < write_blocks && count >= M;
  if (decide) {
    // pairs (i, j) with i < j, plus (i, M) for the candidate
    const int n_pairs = M * (M - 1) / 2 + M;
    for (int p = warp; p < n_pairs; p += nw) {
      int i, j;
      if (p < M * (M - 1) / 2) {
        // unrank p into i < j
        i = 0;
        int rem = p;
        while (rem >= M - 1 - i) { rem -= M - 1 - i; ++i; }
        j = i + 1 + rem;
      } else {
        i = p - M * (M - 1) / 2;
        j = M;
      }
      const float* a = bank_phi + static_cast<size_t>(i) * PRSINK_FP_DIM;
      const float* c = j < M ? bank_phi + static_cast<size_t>(j) * PRSINK_FP_DIM : q;
      const double d = warp_dot(a, c, lane);
      if (lane == 0) {
        G[i][j] = d;
        if (j < M) G[j][i] = d;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int action = -1;
    if (b < write_blocks) {
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
    }
    action_s = action;
    *action_out = action;
    if (action >= 0) {
      bank_src[action] = b;
      if (count < M) *bank_count = count + 1;
    }
  }
  __syncthreads();
  const int a = action_s;
  if (a >= 0)
    for (int i = threadIdx.x; i < PRSINK_FP_DIM; i += blockDim.x)
      bank_phi[static_cast<size_t>(a) * PRSINK_FP_DIM + i] = q[i];
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

extern "C" int prsink_retrieve(const prsink_layout* layout, const float* phi_b,
                               const float* bank_phi, const long long* bank_src,
                               const int* bank_count, int M, long long exclude_block,
                               int* r_out, float* score_out, int* copy_out, long long* dyn_src,
                               const void* bank_kv, void* cache_kv, int n_layers, void* stream) {
  if (!phi_b || !bank_phi || !bank_src || !bank_count || !r_out || !copy_out || !dyn_src) {
    set_error("prsink_retrieve: null pointer");
    return PRSINK_ERR_ARG;
  }
  if (bad_bank(M)) {
    set_error("prsink_retrieve: M = %d outside [1, %d]", M, PRSINK_MAX_BANK);
    return PRSINK_ERR_ARG;
  }
  const bool do_copy = bank_kv || cache_kv || n_layers;
  Geometry g{};
  if (do_copy) {
    int rc = geometry(layout, &g);
    if (rc) return rc;
    if (!bank_kv || !cache_kv || n_layers < 1) {
      set_error("prsink_retrieve: bank_kv, cache_kv and n_layers >= 1 go together");
      return PRSINK_ERR_ARG;
    }
    if (!aligned16(bank_kv) || !aligned16(cache_kv) || (layout->head_dim * 2) % 16) {
      set_error("prsink_retrieve: K/V buffers must be 16-byte aligned");
      return PRSINK_ERR_ALIGN;
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  retrieve_kernel<<<1, 32 * (M < 1 ? 1 : M), 0, st>>>(phi_b, bank_phi, bank_src, bank_count, M,
                                                       exclude_block, r_out, score_out,
                                                       copy_out, dyn_src);
  count_launch();
  int rc = check_launch("prsink_retrieve");
  if (rc || !do_copy) return rc;
  return launch_bank_cache_copy(layout, g, M, n_layers, bank_kv, cache_kv, /*to_cache=*/true,
                                PRSINK_SLOT_DYNAMIC, r_out, copy_out, st);
}

extern "C" int prsink_bank_update(const prsink_layout* layout, float* bank_phi,
                                  long long* bank_src, int* bank_count, int M,
                                  const float* phi_b, long long b, int write_blocks,
                                  int* action_out, const void* cache_kv, void* bank_kv,
                                  int n_layers, void* stream) {
  if (!bank_phi || !bank_src || !bank_count || !phi_b || !action_out) {
    set_error("prsink_bank_update: null pointer");
    return PRSINK_ERR_ARG;
  }
  if (bad_bank(M) || b < 0) {
    set_error("prsink_bank_update: M = %d outside [1, %d] or b = %lld < 0", M, PRSINK_MAX_BANK, b);
    return PRSINK_ERR_ARG;
  }
  const bool do_copy = bank_kv || cache_kv || n_layers;
  Geometry g{};
  if (do_copy) {
    int rc = geometry(layout, &g);
    if (rc) return rc;
    if (!bank_kv || !cache_kv || n_layers < 1) {
      set_error("prsink_bank_update: bank_kv, cache_kv and n_layers >= 1 go together");
      return PRSINK_ERR_ARG;
    }
    if (!aligned16(bank_kv) || !aligned16(cache_kv) || (layout->head_dim * 2) % 16) {
      set_error("prsink_bank_update: K/V buffers must be 16-byte aligned");
      return PRSINK_ERR_ALIGN;
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bank_update_kernel<<<1, 1024, 0, st>>>(bank_phi, bank_src, bank_count, M, phi_b, b,
                                         write_blocks, action_out);
  count_launch();
  int rc = check_launch("prsink_bank_update");
  if (rc || !do_copy) return rc;
  const int ring = PRSINK_SLOT_RING0 + static_cast<int>(b % layout->ring_slots);
  return launch_bank_cache_copy(layout, g, M, n_layers, bank_kv, cache_kv, /*to_cache=*/false,
                                ring, action_out, nullptr, st);
}
