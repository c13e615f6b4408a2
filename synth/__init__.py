"""Seeded synthetic inputs for quantized-KV decode attention.

Shared by the tests and the benchmark; it holds none of the method's
arithmetic (no quantization, no attention), only the workload recipes and a
seeded fp16 generator:

  values      fp16 of N(0,1) draws (torch's seeded generator on the device
              asked for), with chosen K channels multiplied by an outlier
              factor before the fp16 rounding;
  streams     Q, K and V of each (workload, layer) use distinct seeds
              (base seed + 1000*layer + {0: Q, 1: K, 2: V});
  shapes      new K/V rows  [batch][n_tok][n_kv][head_dim]
              queries       [batch][n_q][head_dim]
  projection  the turbo3_qjl key projection: float32 [head_dim][head_dim]
              N(0,1) draws on the host (qjl_projection)

The pages' own workloads (TinyLlama, Llama-3.1-70B and gpt-oss-20b runs)
need trained weights; these synthetic tensors of the same shapes stand in for
them.
"""

from dataclasses import dataclass, field
import math

import torch

TURBO3_SEED = 0x7475726233  # "turb3" in ASCII; any fixed value works


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    layers: int
    n_q: int
    n_kv: int
    head_dim: int
    ctx: int
    k_type: str
    v_type: str
    outlier_channels: tuple
    outlier_scale: float
    seed: int
    turbo_seed: int = 0
    controls: tuple = field(default_factory=tuple)

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    # tiny single decode step: GQA 2, head_dim 64, K channels 3 and 17 x10
    "tiny": Workload("tiny", 1, 1, 4, 2, 64, 256, "q8_0", "q4_0",
                     (3, 17), 10.0, 20260101),
    # Llama-3.1-8B-shaped layer, batch 1, 8K context; f16/f16 and q8_0/q8_0
    # controls on the same inputs
    "llama8b_ctx8k": Workload("llama8b_ctx8k", 1, 1, 32, 8, 128, 8192, "q8_0", "q4_0",
                              (3, 17, 66, 101), 8.0, 20260102,
                              controls=(("f16", "f16"), ("q8_0", "q8_0"))),
    # Llama-3.1-70B-shaped full cache, batch 4, 32K context, K8V4
    "llama70b_ctx32k_b4": Workload("llama70b_ctx32k_b4", 4, 80, 64, 8, 128, 32768, "q8_0", "q4_0",
                                   (3, 17, 66, 101), 8.0, 20260103),
    # long context K4V4 at batch 1 / 4 / 16
    "k4v4_ctx128k_b1": Workload("k4v4_ctx128k_b1", 1, 32, 32, 8, 128, 131072, "q4_0", "q4_0",
                                (3, 17, 66, 101), 8.0, 20260104),
    "k4v4_ctx128k_b4": Workload("k4v4_ctx128k_b4", 4, 32, 32, 8, 128, 131072, "q4_0", "q4_0",
                                (3, 17, 66, 101), 8.0, 20260104),
    "k4v4_ctx128k_b16": Workload("k4v4_ctx128k_b16", 16, 32, 32, 8, 128, 131072, "q4_0", "q4_0",
                                 (3, 17, 66, 101), 8.0, 20260104),
    # TurboQuant-style V: 70B shape, batch 1, 32K, K q8_0 / V turbo3
    "turbo3_ctx32k": Workload("turbo3_ctx32k", 1, 80, 64, 8, 128, 32768, "q8_0", "turbo3",
                              (3, 17, 66, 101), 8.0, 20260105, turbo_seed=TURBO3_SEED),
    # the same at batch 4 (the steady-state rate of the turbo3 value path)
    "turbo3_ctx32k_b4": Workload("turbo3_ctx32k_b4", 4, 80, 64, 8, 128, 32768, "q8_0", "turbo3",
                                 (3, 17, 66, 101), 8.0, 20260105, turbo_seed=TURBO3_SEED),
    # the TurboQuant page's three parts on keys (2-bit levels + 1-bit QJL residual),
    # 70B shape, batch 4, 32K, K turbo3_qjl / V q8_0
    "qjl_ctx32k_b4": Workload("qjl_ctx32k_b4", 4, 80, 64, 8, 128, 32768, "turbo3_qjl", "q8_0",
                              (3, 17, 66, 101), 8.0, 20260106, turbo_seed=TURBO3_SEED),
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_f16(shape, seed, device="cpu", outlier_channels=(), outlier_scale=1.0):
    """fp16 tensor of N(0,1) draws; the listed last-axis channels are
    multiplied by ``outlier_scale`` before rounding to fp16."""
    x = torch.randn(shape, generator=_gen(seed, device), dtype=torch.float32, device=device)
    if outlier_channels:
        idx = torch.tensor(outlier_channels, device=device)
        x[..., idx] *= outlier_scale
    return x.to(torch.float16)


def qjl_projection(seed, head_dim):
    """float32 [head_dim][head_dim] of N(0,1) draws on the host: the random
    projection a turbo3_qjl key cache is coded with (the caller moves it to
    the device for the library; the oracle takes the same host array)."""
    return torch.randn((head_dim, head_dim), generator=_gen(seed, "cpu"), dtype=torch.float32)


def layer_inputs(w: Workload, layer=0, device="cpu", n_tok=None, batch=None):
    """(q, k_new, v_new) fp16 for one layer of workload ``w``.

    q [batch][n_q][head_dim]; k_new, v_new [batch][n_tok][n_kv][head_dim] with
    n_tok = w.ctx unless given.  K carries the outlier channels; Q and V do not.
    """
    b = w.batch if batch is None else batch
    t = w.ctx if n_tok is None else n_tok
    base = w.seed + 1000 * layer
    q = normal_f16((b, w.n_q, w.head_dim), base + 0, device)
    k = normal_f16((b, t, w.n_kv, w.head_dim), base + 1, device,
                   w.outlier_channels, w.outlier_scale)
    v = normal_f16((b, t, w.n_kv, w.head_dim), base + 2, device)
    return q, k, v
