"""Seeded synthetic workloads shaped like Mistral Large 4's sparse-attention layer.

This module only draws random inputs; it contains none of the method's
arithmetic.  Both the CUDA library's tests/bench and the CPU oracle receive the
same tensors from here (copied between device and host), so the two sides never
share code beyond input generation.

Shapes follow the pages: 32 indexer heads x 128, 64 attention heads, a
512-value latent plus a 64-value rotary key per position (512 on NoPE layers),
top 2,048 positions per query.  Distributions and seeds are the stated ones
(bf16 N(0,1) caches and indexer q/k, w ~ N(0,1)/sqrt(32), absorbed queries
~ N(0,1)/sqrt(192) for decode and N(0,1) for prefill, per-(t,h) query
multiplier 1.0 or U(0.5, 1.5)).  The long-context case plants 256 positions per
sequence whose index keys are pushed along the query's head-weighted direction
so the top-k has a clear head and a near-tie tail.

Layout in device memory (shared by every cache buffer):
  rows of sequence b occupy [seq_row_start[b], seq_row_start[b] + L_b)
  k_idx  [rows, 128] bf16        index keys
  cache  [rows, 576 | 512] bf16  [c_s | kR_s] per position, one buffer per layer
  query t belongs to sequence q_seq[t] and sits at position q_pos[t]
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

N_IDX_HEADS = 32
D_IDX = 128
N_HEADS = 64
D_LATENT = 512
D_ROPE = 64
SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)


@dataclass(frozen=True)
class Case:
    """A workload recipe.  kind = "decode" (one query per sequence, at its last
    position) or "prefill" (one sequence: ``cached`` positions already in the
    cache plus ``new`` causal queries whose own rows are appended)."""

    name: str
    kind: str
    seed: int
    lengths: tuple = ()           # decode: context length per sequence
    per_seq: int = 1              # decode: queries per sequence, at its last per_seq positions
    cached: int = 0               # prefill
    new: int = 0                  # prefill
    layers: tuple = (64,)         # d_rope per layer (64 = RoPE, 0 = NoPE)
    qmul: str = "one"             # "one" or "uniform" (U(0.5, 1.5))
    mla_q_std: float = 1.0 / math.sqrt(192.0)
    planted: int = 0              # planted positions per sequence (index keys)
    topk: int = 2048

    @property
    def n_queries(self) -> int:
        return len(self.lengths) * self.per_seq if self.kind == "decode" else self.new

    @property
    def seq_lengths(self) -> tuple:
        return tuple(self.lengths) if self.kind == "decode" else (self.cached + self.new,)

    @property
    def total_rows(self) -> int:
        return sum(self.seq_lengths)

    @property
    def ld(self) -> int:
        """Score-row stride: the longest candidate list, rounded up to 4."""
        return (max(self.seq_lengths) + 3) // 4 * 4


CONFIGS = {
    "tiny_decode": Case(
        name="tiny_decode", kind="decode", seed=0,
        lengths=(4096, 4096, 1500, 37), layers=(64,), qmul="one"),
    "decode_b64_32k": Case(
        name="decode_b64_32k", kind="decode", seed=1,
        lengths=(32768,) * 64, layers=(64,), qmul="uniform"),
    "decode_b16_128k_planted": Case(
        name="decode_b16_128k_planted", kind="decode", seed=2,
        lengths=(131072,) * 16, layers=(64,), qmul="one", planted=256),
    "prefill_32k_plus_8k": Case(
        name="prefill_32k_plus_8k", kind="prefill", seed=3,
        cached=32768, new=8192, layers=(64, 0), qmul="one", mla_q_std=1.0),
    "decode_b4_1m_4layers": Case(
        name="decode_b4_1m_4layers", kind="decode", seed=4,
        lengths=(1 << 20,) * 4, layers=(64, 64, 64, 0), qmul="uniform"),
    # several queries per sequence decoded together (the last 4 positions of each
    # sequence: one token plus 3 drafted ones being verified)
    "decode_b16_32k_4queries": Case(
        name="decode_b16_32k_4queries", kind="decode", seed=5,
        lengths=(32768,) * 16, per_seq=4, layers=(64,), qmul="uniform"),
}


@dataclass
class Layer:
    d_rope: int
    cache: torch.Tensor        # [rows, 512 + d_rope] bf16
    q_nope: torch.Tensor       # [T, 64, 512] bf16
    q_pe: torch.Tensor | None  # [T, 64, 64] bf16, None on NoPE layers
    qmul: torch.Tensor         # [T, 64] f32


@dataclass
class Workload:
    case: Case
    seq_row_start: torch.Tensor   # [B] int64
    q_seq: torch.Tensor           # [T] int32
    q_pos: torch.Tensor           # [T] int32
    q_idx: torch.Tensor           # [T, 32, 128] bf16
    w: torch.Tensor               # [T, 32] f32
    k_idx: torch.Tensor           # [rows, 128] bf16
    layers: list = field(default_factory=list)
    planted_pos: torch.Tensor | None = None   # [B, planted] int64 (positions)

    @property
    def T(self) -> int:
        return int(self.q_seq.shape[0])


def _randn(shape, gen, device, dtype=torch.bfloat16, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _randn_bf16_chunked(rows, cols, gen, device, chunk_rows=1 << 20):
    """bf16 N(0,1) [rows, cols] drawn chunk by chunk to bound fp32 scratch."""
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0, cols), generator=gen, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
    return out


def make_workload(case: Case, device="cpu") -> Workload:
    """Draw every input of ``case`` from torch's generator seeded with case.seed."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(case.seed)

    lens = case.seq_lengths
    starts = [0]
    for L in lens[:-1]:
        starts.append(starts[-1] + L)
    seq_row_start = torch.tensor(starts, dtype=torch.int64, device=device)
    rows = case.total_rows
    if case.kind == "decode":
        m = case.per_seq
        T = len(lens) * m
        q_seq = torch.arange(len(lens), dtype=torch.int32, device=device).repeat_interleave(m)
        q_pos = torch.tensor([L - m + i for L in lens for i in range(m)], dtype=torch.int32, device=device)
    elif case.kind == "prefill":
        T = case.new
        q_seq = torch.zeros(T, dtype=torch.int32, device=device)
        q_pos = torch.arange(case.cached, case.cached + case.new, dtype=torch.int32,
                             device=device)
    else:
        raise ValueError(case.kind)

    k_idx = _randn_bf16_chunked(rows, D_IDX, gen, device)
    q_idx = _randn((T, N_IDX_HEADS, D_IDX), gen, device)
    w = _randn((T, N_IDX_HEADS), gen, device, dtype=torch.float32,
               std=1.0 / math.sqrt(N_IDX_HEADS))

    planted = None
    if case.planted:
        # Push ``planted`` random positions of each sequence along the direction
        # d = sum_j w_j q_j of that sequence's query by 3 standard deviations.
        assert case.kind == "decode" and case.per_seq == 1
        planted = torch.empty((len(lens), case.planted), dtype=torch.int64, device=device)
        for b, L in enumerate(lens):
            pos = torch.randperm(L, generator=gen, device=device)[:case.planted]
            planted[b] = pos.sort().values
            d = (w[b].unsqueeze(1) * q_idx[b].float()).sum(0)
            d = d / d.pow(2).mean().sqrt()
            r = starts[b] + planted[b]
            k_idx[r] = (k_idx[r].float() + 3.0 * d).to(torch.bfloat16)

    layers = []
    for d_rope in case.layers:
        cache = _randn_bf16_chunked(rows, D_LATENT + d_rope, gen, device)
        q_nope = _randn((T, N_HEADS, D_LATENT), gen, device, std=case.mla_q_std)
        q_pe = (_randn((T, N_HEADS, d_rope), gen, device, std=case.mla_q_std)
                if d_rope else None)
        if case.qmul == "uniform":
            qmul = (torch.rand((T, N_HEADS), generator=gen, device=device) + 0.5)
        else:
            qmul = torch.ones((T, N_HEADS), dtype=torch.float32, device=device)
        layers.append(Layer(d_rope=d_rope, cache=cache, q_nope=q_nope, q_pe=q_pe,
                            qmul=qmul.float()))

    return Workload(case=case, seq_row_start=seq_row_start, q_seq=q_seq, q_pos=q_pos,
                    q_idx=q_idx, w=w, k_idx=k_idx, layers=layers, planted_pos=planted)


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row FP8 (E4M3) encoding of an input tensor, for the FP8-key indexer:
    scale = max |x| over the last dimension / 448 (the largest E4M3 value; 1
    for an all-zero row) and codes = e4m3(x / scale) with torch's
    float8_e4m3fn conversion.  Returns (codes uint8 [..., d], scales f32 [...]).
    Input preparation only: both the library and the oracle receive these bytes."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (xf / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


LATENT_FP8_BLOCK = 128


def latent_fp8_row_bytes(d_rope: int, d_c: int = 512) -> int:
    """Bytes per position of an FP8 latent-cache row: the E4M3 codes of
    [c_s | kR_s], one fp32 scale per 128 latent values and one for kR_s (RoPE
    layers), rounded up to a multiple of 16 (608 for RoPE, 528 for NoPE)."""
    n_blk = d_c // LATENT_FP8_BLOCK + (1 if d_rope else 0)
    return (d_c + d_rope + 4 * n_blk + 15) // 16 * 16


def quantize_latent_fp8(cache: torch.Tensor, d_rope: int) -> torch.Tensor:
    """FP8 latent-cache rows from a bf16 cache [rows, >= 512 + d_rope]: per
    128-value block of c_s (and for kR_s as one block) scale = max |x| / 448
    (1 for an all-zero block), codes = e4m3(x / scale) with torch's
    float8_e4m3fn conversion; layout [codes | fp32 scales | zero padding].
    Input preparation only: both the library and the oracle receive these bytes."""
    d_c = 512
    rows = cache.shape[0]
    x = cache[:, :d_c + d_rope].float()
    parts = [x[:, :d_c].reshape(rows, d_c // LATENT_FP8_BLOCK, LATENT_FP8_BLOCK)]
    amax = parts[0].abs().amax(dim=-1)
    if d_rope:
        amax = torch.cat([amax, x[:, d_c:].abs().amax(dim=-1, keepdim=True)], dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    blk_scale = torch.cat([scale[:, :d_c // LATENT_FP8_BLOCK].repeat_interleave(LATENT_FP8_BLOCK, dim=1)] +
                          ([scale[:, -1:].expand(rows, d_rope)] if d_rope else []), dim=1)
    codes = (x / blk_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    out = torch.zeros((rows, latent_fp8_row_bytes(d_rope, d_c)), dtype=torch.uint8, device=cache.device)
    out[:, :d_c + d_rope] = codes
    n_blk = scale.shape[1]
    out[:, d_c + d_rope:d_c + d_rope + 4 * n_blk] = scale.contiguous().view(torch.uint8).reshape(rows, 4 * n_blk)
    return out


def small_case(name, lengths=None, *, kind="decode", cached=0, new=0, layers=(64,),
               qmul="uniform", mla_q_std=1.0 / math.sqrt(192.0), seed=7, topk=2048,
               planted=0, per_seq=1) -> Case:
    """A parity-test recipe with custom sizes (same distributions as above)."""
    return Case(name=name, kind=kind, seed=seed, lengths=tuple(lengths or ()),
                cached=cached, new=new, layers=tuple(layers), qmul=qmul,
                mla_q_std=mla_q_std, planted=planted, topk=topk, per_seq=per_seq)


def to_numpy(x: torch.Tensor):
    """Exact host copy for the oracle: bf16 becomes float32 (exact), ints stay ints."""
    x = x.detach().to("cpu")
    if x.dtype == torch.bfloat16:
        x = x.float()
    return x.numpy()
