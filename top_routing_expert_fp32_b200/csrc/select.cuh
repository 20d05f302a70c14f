// Per-token routing decision from fp32 logits, shared by every router kernel:
// softmax over the E experts, the k largest logits in descending order (equal logits keep the
// lower expert index first), and the gates.
//   Grok-1 book ch.5, 5.2 (softmax, TopK) and 5.2.3 (gates with and without renormalisation);
//   MoE formula-to-code walkthrough 1.1-1.2; LLMs-from-scratch ch.12, 12.1.
#pragma once

#include "common.cuh"

namespace moe {

// z: the token's E logits (shared memory). Writes idx[0..k) and gate[0..k) (global). With
// `probs`, z is overwritten with the full softmax probabilities (for the balance statistic).
//   renorm = 0: gate_j = softmax(z)[idx_j];  renorm = 1: softmax over the selected logits.
// Selection compares logits, never probabilities: softmax is increasing, so the set is the
// same, and the decision is taken in fp32 on the values the caller holds.
__device__ __forceinline__ void select_token(float* z, int E, int k, int renorm, int32_t* idx,
                                             float* gate, bool probs) {
  float zmax = z[0];
  for (int e = 1; e < E; ++e) zmax = z[e] > zmax ? z[e] : zmax;
  uint64_t chosen = 0;
  int sel[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sel[j] = 0;
    if (j < k) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if ((chosen >> e) & 1ull) continue;
        if (best < 0 || z[e] > z[best]) best = e;  // strict: equal keeps the lower index
      }
      chosen |= 1ull << best;
      sel[j] = best;
    }
  }
  float s_all = 0.f;
  for (int e = 0; e < E; ++e) s_all += expf(z[e] - zmax);
  float s_sel = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) s_sel += expf(z[sel[j]] - zmax);
  const float denom = renorm ? s_sel : s_all;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      idx[j] = sel[j];
      gate[j] = expf(z[sel[j]] - zmax) / denom;
    }
  }
  if (probs)
    for (int e = 0; e < E; ++e) z[e] = expf(z[e] - zmax) / s_all;
}

// The same decision with the logits in registers (EB >= E, entries past E ignored): every
// loop is unrolled, so nothing waits on shared memory. Sums run in the same order as
// select_token, so both give the same bits for the same logits. probs (shared memory,
// optional) receives the full softmax.
template <int EB>
__device__ __forceinline__ void select_token_regs(const float (&z)[EB], int E, int k, int renorm,
                                                  int32_t* idx, float* gate, float* probs) {
  float zmax = z[0];
#pragma unroll
  for (int e = 1; e < EB; ++e)
    if (e < E) zmax = z[e] > zmax ? z[e] : zmax;
  uint64_t chosen = 0;
  int sel[8];
  float selz[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sel[j] = 0;
    selz[j] = 0.f;
    if (j < k) {
      int best = -1;
      float zb = 0.f;
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        const bool take = e < E && !((chosen >> e) & 1ull) && (best < 0 || z[e] > zb);
        best = take ? e : best;  // strict: equal keeps the lower index
        zb = take ? z[e] : zb;
      }
      chosen |= 1ull << best;
      sel[j] = best;
      selz[j] = zb;
    }
  }
  float s_all = 0.f;
#pragma unroll
  for (int e = 0; e < EB; ++e)
    if (e < E) s_all += expf(z[e] - zmax);
  float s_sel = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) s_sel += expf(selz[j] - zmax);
  const float denom = renorm ? s_sel : s_all;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      idx[j] = sel[j];
      gate[j] = expf(selz[j] - zmax) / denom;
    }
  }
  if (probs != nullptr) {
#pragma unroll
    for (int e = 0; e < EB; ++e)
      if (e < E) probs[e] = expf(z[e] - zmax) / s_all;
  }
}

}  // namespace moe
