// Per-token routing decision from fp32 logits, shared by every router kernel:
// softmax over the E experts, the k selected experts in order (equal values keep the lower
// expert index first), and the gates.
//   Grok-1 book ch.5, 5.2 (softmax, TopK) and 5.2.3 (gates with and without renormalisation);
//   MoE formula-to-code walkthrough 1.1-1.2; LLMs-from-scratch ch.12, 12.1.
// Training-time variants (mode), with the caller's noise row n:
//   MOE_ROUTE_NOISY_TOPK (Grok-1 book 5.2.2, Switch's noisy top-k): z' = z + n in fp32; the
//     selection and the gates use z'.
//   MOE_ROUTE_GSHARD_RANDOM (MoE series 3): the first expert is the largest z; every later one
//     the largest z' = z + n (fp32) among the experts not chosen yet; the gates use z.
// lse (optional) receives log sum_e exp(z_e) of the unperturbed logits (the z-loss term of
// Grok-1 book 5.2.2).
#pragma once

#include "common.cuh"

namespace moe {

// z: the token's E logits (shared memory). Writes idx[0..k) and gate[0..k) (global). With
// `probs`, z is overwritten with the softmax the gates come from (for the balance statistic).
//   renorm = 0: gate_j = softmax[idx_j];  renorm = 1: softmax over the selected set.
// Selection compares logits, never probabilities: softmax is increasing, so the set is the
// same, and the decision is taken in fp32 on the values the caller holds.
__device__ __forceinline__ void select_token(float* z, int E, int k, int renorm, int mode,
                                             const float* noise, int32_t* idx, float* gate,
                                             bool probs, float* lse) {
  if (lse != nullptr) {
    float m = z[0];
    for (int e = 1; e < E; ++e) m = z[e] > m ? z[e] : m;
    float s = 0.f;
    for (int e = 0; e < E; ++e) s += expf(z[e] - m);
    *lse = m + logf(s);
  }
  if (mode == MOE_ROUTE_NOISY_TOPK)
    for (int e = 0; e < E; ++e) z[e] = z[e] + noise[e];
  float zmax = z[0];
  for (int e = 1; e < E; ++e) zmax = z[e] > zmax ? z[e] : zmax;
  uint64_t chosen = 0;
  int sel[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sel[j] = 0;
    if (j < k) {
      const bool perturbed = mode == MOE_ROUTE_GSHARD_RANDOM && j > 0;
      int best = -1;
      float vb = 0.f;
      for (int e = 0; e < E; ++e) {
        if ((chosen >> e) & 1ull) continue;
        const float v = perturbed ? z[e] + noise[e] : z[e];
        if (best < 0 || v > vb) {  // strict: equal keeps the lower index
          best = e;
          vb = v;
        }
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

}  // namespace moe
