"""Seeded layer cases of the end-to-end parity tests (inputs only, no method arithmetic).

Each case names one weight matrix, its calibration streams and the LB-ADMM settings of
one of the benchmark configurations:

  config 2   Llama-2-7B q_proj 4096 x 4096, 1 % of input columns x10, r = 2032 (1.0 BPW)
  target     the 11008 x 4096 gate/up shape, Student-t(3) column factors, r = 1000
  config 3   Llama-2-7B block at 0.8 BPW: q_proj (r = 1622), gate_proj and down_proj
             (r = 2372), Student-t(3) column factors
  config 4   Llama-2-70B k_proj 1024 x 8192 at 0.55 BPW (r = 484), 0.5 % of columns x8,
             60 iterations
  config 5   one 8192 x 8192 Gaussian matrix without streams (identity preconditioners),
             r in {16, 256, 1024, 4080}, 50 iterations

Ranks are stated as numbers (they follow from the bits-per-weight accounting, which the
oracle's own tests pin).  Calibration streams have the pages' 128 x 2048 = 262144 tokens
(summary page, "Method steps", stage one); weights and streams are BF16.
"""
from dataclasses import dataclass
from typing import Iterator, Optional

import torch

from .inputs import CALIB_TOKENS, gaussian_weight, stream_chunks, student_t_weight


@dataclass(frozen=True)
class Case:
    name: str
    m: int
    n: int
    r: int
    iters: int
    w_kind: str                  # "outlier_cols" or "student_t"
    w_name: str                  # generator key of the weight
    std: float = 0.02
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    act_stream: Optional[str] = None    # None: identity preconditioners
    grad_stream: Optional[str] = None
    T: int = CALIB_TOKENS
    seed: int = 0                # seed of every input generator
    admm_seed: int = 0           # seed of V_0

    def weight(self) -> torch.Tensor:
        if self.w_kind == "student_t":
            return student_t_weight(self.seed, self.w_name, self.m, self.n, self.std, 3)
        return gaussian_weight(self.seed, self.w_name, self.m, self.n, self.std,
                               self.outlier_frac, self.outlier_gain)

    def act_chunks(self) -> Iterator[torch.Tensor]:
        return stream_chunks(self.seed, self.act_stream, self.T, self.n)

    def grad_chunks(self) -> Iterator[torch.Tensor]:
        return stream_chunks(self.seed, self.grad_stream, self.T, self.m)


CASES = {c.name: c for c in [
    Case("c2_q_proj", 4096, 4096, 2032, 100, "outlier_cols", "W", 0.02, 0.01, 10.0,
         "acts", "grads"),
    Case("target_gate_proj", 11008, 4096, 1000, 100, "student_t", "target_gate_proj",
         act_stream="mlp_in", grad_stream="grad_target_gate_proj"),
    Case("c3_q_proj", 4096, 4096, 1622, 100, "student_t", "c3_q_proj",
         act_stream="attn_in", grad_stream="grad_c3_q_proj"),
    Case("c3_gate_proj", 11008, 4096, 2372, 100, "student_t", "c3_gate_proj",
         act_stream="mlp_in", grad_stream="grad_c3_gate_proj"),
    Case("c3_down_proj", 4096, 11008, 2372, 100, "student_t", "c3_down_proj",
         act_stream="down_in", grad_stream="grad_c3_down_proj"),
    Case("c4_k_proj", 1024, 8192, 484, 60, "outlier_cols", "c4_k_proj", 0.015, 0.005, 8.0,
         "attn_in_70b", "grad_c4_k_proj"),
    Case("c5_r16", 8192, 8192, 16, 50, "outlier_cols", "c5_W8192"),
    Case("c5_r256", 8192, 8192, 256, 50, "outlier_cols", "c5_W8192"),
    Case("c5_r1024", 8192, 8192, 1024, 50, "outlier_cols", "c5_W8192"),
    Case("c5_r4080", 8192, 8192, 4080, 50, "outlier_cols", "c5_W8192"),
]}
