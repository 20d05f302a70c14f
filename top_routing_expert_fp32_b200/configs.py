"""Workload shapes for the MoE FFN forward layer.

Each entry is a synthetic workload with the shapes, dtypes and routing options of one layer
described on the pages:

* ``tiny_f32``   -- a small fp32 layer (N=64 tokens as B=2 x T=32, D=64, F=128, E=4, top-2,
  SiLU gating, renormalised top-k, no capacity).
* ``mixtral``    -- Mixtral-shaped: N=4096, D=4096, F=14336, E=8, top-2, SiLU gating, top-k
  renormalised, no capacity (Grok-1 book ch.5, section 5.7; LLMs-from-scratch ch.12 sec 12.1).
* ``grok1``      -- Grok-1-shaped: one 8192-token sequence, d=6144, d_ffn=32768, 8 experts,
  top-2, GELU(x W_gate) * (x W_value) gating, softmax over all 8 then top-2 without
  renormalisation, no capacity (Grok-1 book ch.5, sections 5.2.3 and 5.3.5).
* ``capacity``   -- capacity/drop stress: N=16384, D=2048, F=8192, E=64, k=2 (and k=1),
  CF=1.25, slot-major assignment, per-expert logit bias ~ N(0, variance 2)
  (MoE formula-to-code walkthrough, section 3).
* ``decode``     -- decode-sized, expert-weight-bandwidth-bound: N=64, D=4096, F=14336, E=8,
  top-2, SiLU gating, renormalised.
* ``capacity_gshard`` -- the capacity shape under GShard's policies: token-major positions
  (the walkthrough's dispatch loop, 3.2), the kept slot of a half-dropped token takes the
  whole weight (MoE series 2.2, case A), capacity = max(ceil(CF*N*k/E), min_capacity) with
  CF = 1.0 and min_capacity = 256 (MoE series 2.1).

Only shapes and options live here; no arithmetic of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

DTYPE_F32 = 0
DTYPE_BF16 = 1

ACT_SILU = 0
ACT_GELU_ERF = 1
ACT_GELU_TANH = 2

ORDER_SLOT_MAJOR = 0
ORDER_TOKEN_MAJOR = 1
DROP_ZERO = 0
DROP_RENORM_KEPT = 1

ROUTE_TOPK = 0
ROUTE_NOISY_TOPK = 1
ROUTE_GSHARD_RANDOM = 2


@dataclass(frozen=True)
class MoEConfig:
    name: str
    N: int                      # tokens (B*T flattened)
    D: int                      # model width
    F: int                      # expert FFN width
    E: int                      # experts
    k: int                      # experts per token
    dtype: int                  # DTYPE_F32 or DTYPE_BF16 for X / W1..W3 / outputs
    activation: int             # ACT_*
    renormalize: int            # 1: gates renormalised over the selected set
    capacity_factor: float = 0.0  # <= 0: no capacity
    router_bias_var: float = 0.0  # > 0: per-expert logit bias ~ N(0, var)
    seed: int = 0
    capacity_order: int = ORDER_SLOT_MAJOR
    drop_policy: int = DROP_ZERO
    min_capacity: int = 0
    routing_mode: int = ROUTE_TOPK
    noise_std: float = 0.0          # std of the routing noise (routing_mode != ROUTE_TOPK)

    @property
    def records(self) -> int:
        return self.N * self.k

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


CONFIGS = {
    "tiny_f32": MoEConfig("tiny_f32", N=64, D=64, F=128, E=4, k=2, dtype=DTYPE_F32,
                          activation=ACT_SILU, renormalize=1),
    "mixtral": MoEConfig("mixtral", N=4096, D=4096, F=14336, E=8, k=2, dtype=DTYPE_BF16,
                         activation=ACT_SILU, renormalize=1),
    "grok1": MoEConfig("grok1", N=8192, D=6144, F=32768, E=8, k=2, dtype=DTYPE_BF16,
                       activation=ACT_GELU_ERF, renormalize=0),
    "capacity": MoEConfig("capacity", N=16384, D=2048, F=8192, E=64, k=2, dtype=DTYPE_BF16,
                          activation=ACT_SILU, renormalize=1, capacity_factor=1.25,
                          router_bias_var=2.0),
    "capacity_k1": MoEConfig("capacity_k1", N=16384, D=2048, F=8192, E=64, k=1,
                             dtype=DTYPE_BF16, activation=ACT_SILU, renormalize=1,
                             capacity_factor=1.25, router_bias_var=2.0),
    "decode": MoEConfig("decode", N=64, D=4096, F=14336, E=8, k=2, dtype=DTYPE_BF16,
                        activation=ACT_SILU, renormalize=1),
    "capacity_gshard": MoEConfig("capacity_gshard", N=16384, D=2048, F=8192, E=64, k=2,
                                 dtype=DTYPE_BF16, activation=ACT_SILU, renormalize=1,
                                 capacity_factor=1.0, router_bias_var=2.0,
                                 capacity_order=ORDER_TOKEN_MAJOR,
                                 drop_policy=DROP_RENORM_KEPT, min_capacity=256),
}

# The workload the throughput benchmark times on one GPU.
BENCH_WORKLOAD = "grok1"


def active_ffn_flops(N_kept_records: int, D: int, F: int) -> float:
    """Active expert FLOPs: 2 up-projections + 1 down-projection per kept record
    (parameter accounting of LLMs-from-scratch ch.12 sec 12.3: ~3*D*F weights per expert)."""
    return 6.0 * N_kept_records * D * F
