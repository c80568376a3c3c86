"""The synthetic workloads of the routed-MoE expert pass.

Model shapes follow the pages: 48 layers of 512 routed experts, 10 routed + 1
shared expert per token (wiselychen RTX 5090 report, "30 秒定位"; greenbean-ai
"Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next", §一).  Expert width d_model =
3072, d_ff = 512 and the block formats are readings (the pages give neither).

  tiny        1 layer, D=256, F=128, E=16, top-2 + shared, 4 tokens, Q2_32, all resident
  decode      1 layer, D=3072, F=512, E=512, top-10 + shared, 4 tokens (1 + 3 MTP drafts),
              Q2_32, 320 of 512 experts resident, Zipf(1.1) router bias (~93% hits; the
              wiselychen report §2 quotes a 93.4% GPU expert-cache hit rate)
  decode48    48 layers of decode shapes, 1 token, Q3_32, 7,948 resident slots over the
              layers (tutuge.me 4090 report: 7,948 slots, 95.6-97.8% hits), per-layer
              Zipf(1.1) popularity; layer input = previous output + residual
  prefill     1 layer, 2,048 tokens, Q2_32, all resident, Zipf(0.8) router bias
              (expert loads from 0 to ~1,450 tokens)
  prefill48   48 layers x 4,096 tokens, Q3_S256, all resident (~50 GB of experts),
              no bias (uniform routing), layer input = previous output + residual
  decode_coder, prefill_coder
              the "Coder" shape: 256 of the 512 routed experts kept per layer
              (greenbean-ai §四, the Coder checkpoint), otherwise the decode and
              prefill workloads' shapes, routing and bias; all 256 experts resident
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

from . import synth


@dataclass(frozen=True)
class Config:
    name: str
    layers: int
    D: int
    F: int
    E: int
    k: int
    T: int
    fmt: int
    resident_per_layer: Optional[List[int]]   # None: all E experts resident
    zipf_s: Optional[float]
    zipf_alpha: Optional[float]
    seed: int = 0
    chained: bool = False
    # Weight std of the synthetic experts.  The pass has no normalisation, and a
    # SwiGLU expert responds quadratically to its input: a 48-layer residual
    # chain stays bounded (|x| ~ 4) at std <= ~0.01 but diverges at 0.02+.
    weight_std: float = 0.02


def _split_slots(total: int, layers: int) -> List[int]:
    base, extra = divmod(total, layers)
    return [base + (1 if l < extra else 0) for l in range(layers)]


CONFIGS = {
    # seed 1: every token's k-th and (k+1)-th logits differ by >= 1e-2 (pinned by a test)
    "tiny": Config("tiny", 1, 256, 128, 16, 2, 4, synth.Q2_32, None, None, None, seed=1),
    "decode": Config("decode", 1, 3072, 512, 512, 10, 4, synth.Q2_32, [320], 1.1, 0.47),
    "decode48": Config("decode48", 48, 3072, 512, 512, 10, 1, synth.Q3_32,
                       _split_slots(7948, 48), 1.1, 0.75, chained=True, weight_std=0.008),
    "prefill": Config("prefill", 1, 3072, 512, 512, 10, 2048, synth.Q2_32, None, 0.8, 0.8),
    "prefill48": Config("prefill48", 48, 3072, 512, 512, 10, 4096, synth.Q3_S256, None, None, None,
                        chained=True, weight_std=0.008),
}
CONFIGS["decode_coder"] = Config("decode_coder", 1, 3072, 512, 256, 10, 4, synth.Q2_32, None, 1.1, 0.47)
CONFIGS["prefill_coder"] = Config("prefill_coder", 1, 3072, 512, 256, 10, 2048, synth.Q2_32, None, 0.8, 0.8)
ORDER = ["tiny", "decode", "decode48", "prefill", "prefill48", "decode_coder", "prefill_coder"]


@dataclass
class Layer:
    Wr: torch.Tensor            # bf16 [E, D]
    bias: Optional[torch.Tensor]  # fp32 [E] or None
    slot_table: torch.Tensor    # int32 [E]
    shared_slot: int


@dataclass
class Workload:
    cfg: Config
    pool: synth.PoolData
    layers: List[Layer] = field(default_factory=list)
    x: Optional[torch.Tensor] = None   # bf16 [T, D], the first layer's input

    @property
    def n_resident(self) -> int:
        return sum(int((l.slot_table >= 0).sum()) for l in self.layers)


def build(cfg: Config, device="cpu", T: Optional[int] = None, layers: Optional[int] = None,
          pool_device=None) -> Workload:
    """Generate the workload: one pool holding every layer's resident experts and
    shared expert, per-layer router weights, biases and slot tables, and x."""
    L = cfg.layers if layers is None else layers
    T = cfg.T if T is None else T
    E = cfg.E
    resident = [E] * L if cfg.resident_per_layer is None else list(cfg.resident_per_layer[:L])
    n_slots = sum(resident) + L                      # + one shared expert per layer
    pool = synth.make_pool(cfg.fmt, cfg.D, cfg.F, n_slots, cfg.seed,
                           device=pool_device or device, weight_std=cfg.weight_std)
    # global slot placement: a seeded permutation of all slots
    perm = synth.slot_permutation(n_slots, cfg.seed)
    wl = Workload(cfg, pool)
    pos = 0
    for l in range(L):
        order = synth.popularity_order(E, cfg.seed, l)
        res = order[:resident[l]]
        st = synth.slot_table(E, res, perm[pos:pos + resident[l]])
        pos += resident[l]
        shared = int(perm[pos]); pos += 1
        bias = None
        if cfg.zipf_s is not None:
            bias = synth.zipf_bias(E, cfg.zipf_s, cfg.zipf_alpha, cfg.seed, l).to(device)
        wl.layers.append(Layer(synth.router_weight(E, cfg.D, cfg.seed, l, device=device), bias,
                               st.to(device), shared))
    wl.x = synth.hidden(T, cfg.D, cfg.seed, device=device)
    return wl
