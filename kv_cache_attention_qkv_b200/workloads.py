"""Seeded synthetic inputs for one Flash-Cache step.

This module only draws random numbers and lays them out; it holds none of the
step's arithmetic, so both the CPU oracle and the CUDA path can be fed from it.

Five workloads are defined, named by what they are:

* ``tiny_fp32``      B=1, hidden 32, 2 heads x 16, theta 1e4, cache 64, fp32.
                     Window at 40..43, 4 tracked positions drawn from 0..39.
* ``layer_b1``       B=1, hidden 4096, 32 heads x 128, theta 5e5, cache 768
                     (256 prompt + 512 generated), 64 tracked + 64 window, bf16.
* ``batch32_uniform`` B=32, same layer, cache 1536 (1024 + 512) per sequence,
                     64 tracked + 64 window, bf16.  The headline workload.
* ``batch32_varlen`` B=32, same layer, cache length U[600, 2048] per sequence,
                     window 16 or 64 and tracking budget 48/64/80 per sequence.
* ``small_varlen``   a few-second ragged case for element-wise parity: B=3,
                     hidden 256, 4 heads x 128, caches of 129..700 rows.
* ``small_d64``      bf16 with head_dim 64 (the CUDA-core path): B=2, hidden
                     96, 3 heads x 64, caches of 200 and 333 rows.
* ``small_longcache`` the small_varlen layer with caches of 2049, 2048, 700
                     and 129 rows: ragged key tiles over the longest caches of
                     the element-wise parity cases.

Sweep points are named ``sweep_b<B>_m<beta>_L<L>``: the headline recipe with
B sequences, a query of beta rows (beta/2 tracked + a beta/2-row window) and a
cache of L rows per sequence (the generated span is the last 512 rows, or the
last half of the cache when it is shorter).  They mirror the axes the pages
measure (batch size, query size beta_m, cache length).

The shapes follow LLaDA-8B (the model the Flash-dLLM pages evaluate); weights
and caches are random, there is no dataset and no checkpoint.

Every bf16 tensor is drawn in fp32 and rounded to bf16 by torch; the fp32 copy
returned alongside holds exactly the bf16 values, so both sides start from the
same numbers.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

WORKLOADS = ("tiny_fp32", "layer_b1", "batch32_uniform", "batch32_varlen", "small_varlen",
             "small_d64", "small_longcache")


@dataclasses.dataclass
class StepInputs:
    """One step's inputs.  Float arrays are fp32 numpy holding dtype-exact values."""

    name: str
    dtype: str  # "bf16" or "fp32"
    hidden: int
    n_heads: int
    head_dim: int
    rope_theta: float
    x: np.ndarray  # [T, hidden]
    w_qkv: np.ndarray  # [3*H*d, hidden]; rows = [Q heads | K heads | V heads]
    k_cache: np.ndarray  # [S, H, d] (prior contents)
    v_cache: np.ndarray  # [S, H, d]
    q_pos: np.ndarray  # int32 [T], absolute positions inside each sequence
    cu_seqlens_q: np.ndarray  # int32 [B+1]
    cu_seqlens_k: np.ndarray  # int32 [B+1]
    cand_lo: np.ndarray  # int32 [B], candidate positions for reselection
    cand_hi: np.ndarray  # int32 [B]
    topk: np.ndarray  # int32 [B], tracking budget per sequence
    window_start: np.ndarray  # int32 [B]
    window_len: np.ndarray  # int32 [B]

    @property
    def batch(self) -> int:
        return int(self.cu_seqlens_q.shape[0] - 1)

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def total_k(self) -> int:
        return int(self.cu_seqlens_k[-1])

    @property
    def max_topk(self) -> int:
        return int(self.topk.max())

    def seq_slice_q(self, b: int) -> slice:
        return slice(int(self.cu_seqlens_q[b]), int(self.cu_seqlens_q[b + 1]))

    def seq_slice_k(self, b: int) -> slice:
        return slice(int(self.cu_seqlens_k[b]), int(self.cu_seqlens_k[b + 1]))


def to_bf16_exact(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 with torch and return them widened to fp32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _layout(rng, lens_k: List[int], windows: List[int], budgets: List[int],
            window_starts: List[int]):
    """Query = tracked positions (ascending) then the masked window (ascending)."""
    pos_rows = []
    for L, w, kb, ws in zip(lens_k, windows, budgets, window_starts):
        assert kb <= ws and ws + w <= L
        tracked = np.sort(rng.choice(ws, size=kb, replace=False)).astype(np.int32)
        window = np.arange(ws, ws + w, dtype=np.int32)
        pos_rows.append(np.concatenate([tracked, window]))
    n = [len(p) for p in pos_rows]
    cu_q = np.zeros(len(n) + 1, np.int32)
    cu_q[1:] = np.cumsum(n)
    cu_k = np.zeros(len(lens_k) + 1, np.int32)
    cu_k[1:] = np.cumsum(lens_k)
    return np.concatenate(pos_rows).astype(np.int32), cu_q, cu_k


def parse_sweep(name: str):
    """(B, beta, L) of a ``sweep_b<B>_m<beta>_L<L>`` name, else None."""
    import re

    m = re.fullmatch(r"sweep_b(\d+)_m(\d+)_L(\d+)", name)
    if not m:
        return None
    B, beta, L = (int(v) for v in m.groups())
    if B < 1 or beta < 2 or beta % 2 or L < 2 * beta:
        raise ValueError(f"bad sweep point {name!r}: need B >= 1, even beta >= 2, L >= 2 beta")
    return B, beta, L


def generate(name: str, seed: Optional[int] = None, batch: Optional[int] = None) -> StepInputs:
    """Draw the named workload.  ``seed`` defaults to the workload's index.

    ``batch`` overrides the number of sequences (used to draw a sub-sample or a
    per-rank shard of the same recipe); per-sequence draws keep their recipe.
    """
    sweep = parse_sweep(name)
    if name not in WORKLOADS and sweep is None:
        raise ValueError(f"unknown workload {name!r}; known: {WORKLOADS} and sweep_b<B>_m<beta>_L<L>")
    if seed is None:
        seed = WORKLOADS.index(name) if sweep is None else 100
    rng = np.random.default_rng(seed)

    if sweep is not None:
        dtype, D, H, d, theta, w_std = "bf16", 4096, 32, 128, 5.0e5, 0.02
        B0, beta, L = sweep
        B = batch or B0
        half = beta // 2
        gen = min(512, L // 2)  # generated span: the last `gen` rows of the cache
        lens = [L] * B
        windows = [half] * B
        budgets = [half] * B
        n_slots = (gen - half) // half + 1
        starts = [int(L - gen + half * rng.integers(0, n_slots)) for _ in range(B)]
    elif name == "tiny_fp32":
        dtype, D, H, d, theta, w_std = "fp32", 32, 2, 16, 1.0e4, 0.1
        B = batch or 1
        lens = [64] * B
        windows = [4] * B
        budgets = [4] * B
        starts = [40] * B
    elif name == "layer_b1":
        dtype, D, H, d, theta, w_std = "bf16", 4096, 32, 128, 5.0e5, 0.02
        B = batch or 1
        lens = [768] * B
        windows = [64] * B
        budgets = [64] * B
        # 64-aligned window inside the generated span [256, 768)
        starts = [int(256 + 64 * rng.integers(0, (768 - 256) // 64)) for _ in range(B)]
    elif name == "batch32_uniform":
        dtype, D, H, d, theta, w_std = "bf16", 4096, 32, 128, 5.0e5, 0.02
        B = batch or 32
        lens = [1536] * B
        windows = [64] * B
        budgets = [64] * B
        starts = [int(1024 + 64 * rng.integers(0, (1536 - 1024) // 64)) for _ in range(B)]
    elif name == "batch32_varlen":
        dtype, D, H, d, theta, w_std = "bf16", 4096, 32, 128, 5.0e5, 0.02
        B = batch or 32
        lens = [int(v) for v in rng.integers(600, 2049, size=B)]
        windows = [int(v) for v in rng.choice([16, 64], size=B)]
        budgets = [int(v) for v in rng.choice([48, 64, 80], size=B)]
        starts = []
        for L, w, kb in zip(lens, windows, budgets):
            lo = L - min(512, L - kb)
            first = -(-lo // w) * w
            last = L - w
            starts.append(int(first + w * rng.integers(0, (last - first) // w + 1)))
    elif name == "small_d64":
        dtype, D, H, d, theta, w_std = "bf16", 96, 3, 64, 1.0e4, 0.1
        B = batch or 2
        lens = [[200, 333][i % 2] for i in range(B)]
        windows = [[16, 64][i % 2] for i in range(B)]
        budgets = [[40, 64][i % 2] for i in range(B)]
        starts = [[48, 256][i % 2] for i in range(B)]
    elif name == "small_longcache":
        dtype, D, H, d, theta, w_std = "bf16", 256, 4, 128, 5.0e5, 0.0625
        B = batch or 4
        lens = [[2049, 2048, 700, 129][i % 4] for i in range(B)]
        windows = [[64, 16, 64, 16][i % 4] for i in range(B)]
        budgets = [[80, 48, 100, 48][i % 4] for i in range(B)]
        starts = []
        for L, w, kb in zip(lens, windows, budgets):
            first = -(-kb // w) * w
            starts.append(int(first + w * rng.integers(0, (L - w - first) // w + 1)))
    else:  # small_varlen
        dtype, D, H, d, theta, w_std = "bf16", 256, 4, 128, 5.0e5, 0.0625
        B = batch or 3
        base_lens = [700, 129, 333]
        lens = [base_lens[i % 3] for i in range(B)]
        windows = [64, 16, 64]
        windows = [windows[i % 3] for i in range(B)]
        budgets = [80, 48, 100]
        budgets = [budgets[i % 3] for i in range(B)]
        starts = []
        for L, w, kb in zip(lens, windows, budgets):
            first = -(-kb // w) * w
            starts.append(int(first + w * rng.integers(0, (L - w - first) // w + 1)))

    q_pos, cu_q, cu_k = _layout(rng, lens, windows, budgets, starts)
    T, S = int(cu_q[-1]), int(cu_k[-1])

    x = _normal(rng, (T, D), 1.0)
    w = _normal(rng, (3 * H * d, D), w_std)
    kc = _normal(rng, (S, H, d), 1.0)
    vc = _normal(rng, (S, H, d), 1.0)
    if dtype == "bf16":
        x, w, kc, vc = (to_bf16_exact(a) for a in (x, w, kc, vc))

    starts_a = np.asarray(starts, np.int32)
    return StepInputs(
        name=name, dtype=dtype, hidden=D, n_heads=H, head_dim=d, rope_theta=float(theta),
        x=x, w_qkv=w, k_cache=kc, v_cache=vc, q_pos=q_pos,
        cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
        cand_lo=np.zeros(B, np.int32), cand_hi=starts_a.copy(),
        topk=np.asarray(budgets, np.int32), window_start=starts_a,
        window_len=np.asarray(windows, np.int32),
    )


def describe(name: str) -> Dict[str, object]:
    """Shape summary of a workload without drawing its tensors."""
    table = {
        "tiny_fp32": dict(dtype="fp32", B=1, hidden=32, heads=2, head_dim=16, cache="64",
                          query="4 tracked + 4 window"),
        "layer_b1": dict(dtype="bf16", B=1, hidden=4096, heads=32, head_dim=128, cache="768",
                         query="64 tracked + 64 window"),
        "batch32_uniform": dict(dtype="bf16", B=32, hidden=4096, heads=32, head_dim=128,
                                cache="1536", query="64 tracked + 64 window"),
        "batch32_varlen": dict(dtype="bf16", B=32, hidden=4096, heads=32, head_dim=128,
                               cache="U[600,2048]", query="48/64/80 tracked + 16/64 window"),
        "small_varlen": dict(dtype="bf16", B=3, hidden=256, heads=4, head_dim=128,
                             cache="700,129,333", query="80+64, 48+16, 100+64"),
        "small_d64": dict(dtype="bf16", B=2, hidden=96, heads=3, head_dim=64,
                          cache="200,333", query="40+16, 64+64"),
        "small_longcache": dict(dtype="bf16", B=4, hidden=256, heads=4, head_dim=128,
                             cache="2049,2048,700,129", query="80+64, 48+16, 100+64, 48+16"),
    }
    return table[name]


# --------------------------------------------------------------------------
# Model-step inputs (the decoder stack around the Flash-Cache layer)

MODEL_WORKLOADS = ("model_small", "model_llada8b")


@dataclasses.dataclass
class ModelInputs:
    """One model step's inputs, drawn directly on a torch device (bf16).

    ``x_mask`` and ``x_draft`` are the two Flash-Verify views of the query
    rows: the tracked rows are the same in both; the window rows are one
    shared [MASK] vector in the first and one vector per row (the drafts) in
    the second.  ``head_rows`` are the packed indices of the window rows, the
    rows the LM head scores.
    """

    name: str
    hidden: int
    n_heads: int
    head_dim: int
    rope_theta: float
    intermediate: int
    vocab: int
    n_layers: int
    layers: list  # per layer: dict of bf16 tensors (fc_layer_weights names)
    final_norm: object
    lm_head: object
    x_mask: object
    x_draft: object
    embed: object  # [V, D] token embeddings (for decoding); the [MASK] token is V - 1
    k_caches: list
    v_caches: list
    q_pos: np.ndarray
    cu_seqlens_q: np.ndarray
    cu_seqlens_k: np.ndarray
    head_rows: np.ndarray
    cand_lo: np.ndarray
    cand_hi: np.ndarray
    topk: np.ndarray
    window_start: np.ndarray
    window_len: np.ndarray

    @property
    def batch(self) -> int:
        return int(self.cu_seqlens_q.shape[0] - 1)

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def total_k(self) -> int:
        return int(self.cu_seqlens_k[-1])


def generate_model(name: str, device="cuda", seed: Optional[int] = None) -> ModelInputs:
    """Draw a model workload on ``device`` with a seeded torch generator.

    * ``model_small``: 2 layers, hidden 256, 2 heads x 128, SwiGLU 512, vocab
      1000 (a ragged last vocabulary tile), B=2 with caches of 300 and 200 rows,
      24/16 tracked + 16 window rows; weights N(0, 0.0625).
    * ``model_llada8b``: the LLaDA-8B shapes of the pages' model (32 layers,
      hidden 4096, 32 heads x 128, SwiGLU 12288, vocab 126464), B=32, caches
      of 1536 rows, 64 tracked + 64 window rows; weights N(0, 0.02).
    Norm weights are 1 + N(0, 0.1); prior caches N(0, 1); input rows N(0, 1).
    """
    import torch

    if name not in MODEL_WORKLOADS:
        raise ValueError(f"unknown model workload {name!r}; known: {MODEL_WORKLOADS}")
    if seed is None:
        seed = 200 + MODEL_WORKLOADS.index(name)
    rng = np.random.default_rng(seed)
    if name == "model_small":
        D, H, d, I, V, NL, theta, w_std = 256, 2, 128, 512, 1000, 2, 5.0e5, 0.0625
        lens, windows, budgets = [300, 200], [16, 16], [24, 16]
        starts = [208, 160]
    else:
        D, H, d, I, V, NL, theta, w_std = 4096, 32, 128, 12288, 126464, 32, 5.0e5, 0.02
        B = 32
        lens, windows, budgets = [1536] * B, [64] * B, [64] * B
        starts = [int(1024 + 64 * rng.integers(0, (1536 - 1024) // 64)) for _ in range(B)]
    q_pos, cu_q, cu_k = _layout(rng, lens, windows, budgets, starts)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    head_rows = np.concatenate([np.arange(cu_q[b + 1] - w, cu_q[b + 1])
                                for b, w in enumerate(windows)]).astype(np.int32)

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    bf = torch.bfloat16

    def normal(shape, std):
        return (torch.randn(shape, generator=gen, device=device) * std).to(bf)

    def norm_w():
        return (1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)).to(bf)

    layers = []
    for _ in range(NL):
        layers.append({"attn_norm": norm_w(), "w_qkv": normal((3 * H * d, D), w_std),
                       "w_o": normal((D, H * d), w_std), "mlp_norm": norm_w(),
                       "w_gate": normal((I, D), w_std), "w_up": normal((I, D), w_std),
                       "w_down": normal((D, I), w_std)})
    final_norm = norm_w()
    lm_head = normal((V, D), w_std)
    x_draft = normal((T, D), 1.0)
    x_mask = x_draft.clone()
    mask_vec = normal((D,), 1.0)
    x_mask[torch.from_numpy(head_rows).long().to(device)] = mask_vec
    embed = normal((V, D), 1.0)
    k_caches = [normal((S, H, d), 1.0) for _ in range(NL)]
    v_caches = [normal((S, H, d), 1.0) for _ in range(NL)]
    starts_a = np.asarray(starts, np.int32)
    return ModelInputs(
        name=name, hidden=D, n_heads=H, head_dim=d, rope_theta=float(theta), intermediate=I,
        vocab=V, n_layers=NL, layers=layers, final_norm=final_norm, lm_head=lm_head,
        x_mask=x_mask, x_draft=x_draft, embed=embed, k_caches=k_caches, v_caches=v_caches,
        q_pos=q_pos,
        cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, head_rows=head_rows,
        cand_lo=np.zeros(len(lens), np.int32), cand_hi=starts_a.copy(),
        topk=np.asarray(budgets, np.int32), window_start=starts_a,
        window_len=np.asarray(windows, np.int32))
