"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws inputs.  It holds none of the method's arithmetic
(no scores, no selection, no attention) and imports neither the CUDA
library nor the oracle, so both sides can take their inputs from it.

Recipes (the pages give no data; these stand in for the workloads they
describe):

* ``structured_indexer``: adjacent layers share a low-rank token latent so
  their top-k selections overlap, as the pages report (70%-100%).  A token
  latent Z ~ N(0,1)^{L x r} and projections A_h, A_k ~ N(0,1)^{r x d}/sqrt(r)
  are shared by all layers; layer l adds its own noise:
      q_I[t,h] = base_std * Z[t] A_h + noise_std * eps,   k_I[s] likewise,
  rounded once to bf16.  w ~ U(0,1) is drawn once and shared by the
  layers of a group: with a fresh w per layer the adjacent-layer overlap
  stays near 60% whatever the noise, below the pages' band.  The layer
  noise defaults to 0.2 (0.3 gave 65-68% at H_I=32..64, d_I=128).
* ``attention_inputs``: Q, K, V ~ N(0,1) bf16, drawn per layer.
* ``quantize_e4m3_rows``: per-row scaled fp8 e4m3 codes (scale = amax/448,
  1 for a zero row), via torch's own float8_e4m3fn cast.  This is input
  preparation for the fp8 indexer, whose inputs are codes plus scales.

Every tensor is drawn from its own generator seeded by ``seed_for`` over a
(name, layer, tensor) tuple, so any tensor can be re-drawn alone.
"""

from __future__ import annotations

import hashlib

import torch


def seed_for(*parts) -> int:
    """Stable 63-bit seed from a tuple of names and numbers."""
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, seed: int, device="cpu", std: float = 1.0, dtype=torch.float32) -> torch.Tensor:
    x = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def uniform(shape, seed: int, device="cpu", lo: float = 0.0, hi: float = 1.0) -> torch.Tensor:
    x = torch.rand(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.mul_(hi - lo).add_(lo)


class StructuredIndexer:
    """Per-layer indexer inputs with a shared low-rank token structure.

    ``layer(l)`` returns (q_I [B, L, H, d] bf16, k_I [B, L, d] bf16, w [B, L, H] fp32).
    ``keys(l)`` returns that layer's k_I alone (the same values); ``queries(l, t0, t1)``
    draws the query rows t0..t1-1 of the same recipe without building the full
    query tensor (its noise is its own draw, so it is not a slice of ``layer``'s q_I).
    The shared factors are built once per instance (fp32, on ``device``).
    """

    def __init__(self, name: str, B: int, L: int, H: int, d: int, r: int,
                 base_std: float, noise_std: float, device="cpu", seed: int = 0):
        self.name, self.B, self.L, self.H, self.d = name, B, L, H, d
        self.noise_std, self.device, self.seed = noise_std, device, seed
        self.z = normal((B, L, r), seed_for(seed, name, "Z"), device)
        self.a_q = normal((H, r, d), seed_for(seed, name, "A_q"), device, std=base_std / r ** 0.5)
        a_k = normal((r, d), seed_for(seed, name, "A_k"), device, std=base_std / r ** 0.5)
        self.base_k = (self.z @ a_k).contiguous()
        self.w = uniform((B, L, H), seed_for(seed, name, "w"), device)

    def _base_q(self, t0: int, t1: int) -> torch.Tensor:
        # base_q[b,t,h,:] = Z[b,t] @ A_q[h]
        return torch.einsum("btr,hrd->bthd", self.z[:, t0:t1], self.a_q).contiguous()

    def layer(self, l: int):
        B, L, H, d = self.B, self.L, self.H, self.d
        q = normal((B, L, H, d), seed_for(self.seed, self.name, l, "q_noise"), self.device, std=self.noise_std)
        q.add_(self._base_q(0, L))
        q = q.to(torch.bfloat16)
        return q, self.keys(l), self.w

    def keys(self, l: int) -> torch.Tensor:
        B, L, d = self.B, self.L, self.d
        k = normal((B, L, d), seed_for(self.seed, self.name, l, "k_noise"), self.device, std=self.noise_std)
        k.add_(self.base_k)
        return k.to(torch.bfloat16)

    def queries(self, l: int, t0: int, t1: int):
        """(q_I [B, t1-t0, H, d] bf16, w [B, t1-t0, H] fp32) for positions t0..t1-1."""
        B, H, d = self.B, self.H, self.d
        q = normal((B, t1 - t0, H, d), seed_for(self.seed, self.name, l, "q_rows", t0, t1), self.device,
                   std=self.noise_std)
        q.add_(self._base_q(t0, t1))
        return q.to(torch.bfloat16), self.w[:, t0:t1].contiguous()


class SegmentedIndexer:
    """Indexer inputs of a layer group whose layers fall into segments: the layers of one
    segment share one StructuredIndexer's token structure and head weights (their top-k
    selections overlap strongly), while each segment draws its own (selections of layers in
    different segments barely overlap).  A stand-in for a model whose layers change what they
    attend to at a few depths, the case a search over F/S patterns has to find.
    ``segment_starts`` lists the first layer of each segment and starts with 0."""

    def __init__(self, name: str, B: int, L: int, H: int, d: int, r: int, base_std: float, noise_std: float,
                 segment_starts, device="cpu", seed: int = 0):
        starts = list(segment_starts)
        assert starts and starts[0] == 0 and starts == sorted(set(starts))
        self.starts = starts
        self.parts = [StructuredIndexer(f"{name}/segment{i}", B, L, H, d, r, base_std, noise_std, device, seed)
                      for i in range(len(starts))]

    def segment(self, l: int) -> int:
        return max(i for i, s in enumerate(self.starts) if s <= l)

    def layer(self, l: int):
        return self.parts[self.segment(l)].layer(l)


def attention_inputs(name: str, l: int, B: int, L_q: int, L_kv: int, Hq: int, Hkv: int,
                     d_qk: int, d_v: int | None, device="cpu", seed: int = 0):
    """Q [B, L_q, Hq, d_qk], K [B, L_kv, Hkv, d_qk], V [B, L_kv, Hkv, d_v] (None if d_v is None), bf16."""
    Q = normal((B, L_q, Hq, d_qk), seed_for(seed, name, l, "Q"), device, dtype=torch.bfloat16)
    K = normal((B, L_kv, Hkv, d_qk), seed_for(seed, name, l, "K"), device, dtype=torch.bfloat16)
    V = None
    if d_v is not None:
        V = normal((B, L_kv, Hkv, d_v), seed_for(seed, name, l, "V"), device, dtype=torch.bfloat16)
    return Q, K, V


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row (last dim) scaled e4m3: returns (codes uint8, scale fp32 [...]).

    scale = max|x| / 448 (1 for an all-zero row); codes = e4m3(x / scale)
    with round-to-nearest-even (torch's float8_e4m3fn cast), clamped to
    +-448 first so no value can reach the NaN code.
    """
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (xf / scale.unsqueeze(-1)).clamp_(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def integer_indexer(name: str, B: int, L: int, H: int, d: int, lo: int, hi: int, seed: int = 0,
                    w_steps: int = 4, q_rows: int | None = None):
    """Indexer inputs whose scores are exact in fp32 whatever the summation order:
    q_I [B, L, H, d] and k_I [B, L, d] hold integers drawn uniformly from lo..hi (exact in
    bf16), w [B, L, H] holds multiples of 1/w_steps in [0, 1].  With |lo|, |hi| <= 8 and
    d <= 128 every dot product is an integer of magnitude <= 8192 and every partial sum over
    heads a multiple of 1/w_steps well inside fp32's 24-bit significand, so any two correct
    implementations produce identical scores and, with ties to the lower index, identical
    selections.  Small ranges give many equal scores (ties) and many zero scores (ReLU).
    ``q_rows``: draw only that many query rows (q_I and w of the last q_rows positions; a
    decode step needs one row against a long key cache)."""
    nq = L if q_rows is None else q_rows

    def ints(shape, tag):
        g = _gen(seed_for(seed, name, tag), "cpu")
        return torch.randint(lo, hi + 1, shape, generator=g, dtype=torch.int32)

    q = ints((B, nq, H, d), "q").to(torch.bfloat16)
    k = ints((B, L, d), "k").to(torch.bfloat16)
    g = _gen(seed_for(seed, name, "w"), "cpu")
    w = torch.randint(0, w_steps + 1, (B, nq, H), generator=g, dtype=torch.int32).to(torch.float32) / w_steps
    return q.contiguous(), k.contiguous(), w.contiguous()


def integer_indexer_e4m3(name: str, B: int, L: int, H: int, d: int, lo: int, hi: int, seed: int = 0,
                         q_rows: int | None = None):
    """fp8 counterpart of ``integer_indexer``: E4M3 codes of integers lo..hi (every integer of
    magnitude <= 16 is an E4M3 value), per-row scales that are powers of two (2^-3 .. 2^1), and
    w in multiples of 1/4.  Returns (q8 uint8 [B,L,H,d], q_scale fp32 [B,L,H], k8 uint8 [B,L,d],
    k_scale fp32 [B,L], w fp32 [B,L,H]); scores of the real values code x scale stay exact in
    fp32.  ``q_rows`` as for ``integer_indexer``."""
    nq = L if q_rows is None else q_rows

    def ints(shape, tag, a, b):
        g = _gen(seed_for(seed, name, tag), "cpu")
        return torch.randint(a, b + 1, shape, generator=g, dtype=torch.int32)

    q8 = ints((B, nq, H, d), "q8", lo, hi).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = ints((B, L, d), "k8", lo, hi).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    q_scale = torch.exp2(ints((B, nq, H), "q_scale", -3, 1).to(torch.float32))
    k_scale = torch.exp2(ints((B, L), "k_scale", -3, 1).to(torch.float32))
    w = ints((B, nq, H), "w", 0, 4).to(torch.float32) / 4
    return q8.contiguous(), q_scale.contiguous(), k8.contiguous(), k_scale.contiguous(), w.contiguous()
