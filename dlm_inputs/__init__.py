"""Seeded synthetic inputs for the diffusion-LM noising-plus-loss path.

This module holds no arithmetic of the method: it only draws clean token ids,
logits, hidden states, head weights and packed-document lengths from torch's
seeded generators, with the shapes and value distributions of the workloads
the pages train on.  The CPU oracle and the CUDA path both consume what it
returns; neither is imported here.

Shapes follow the pages:
  * vocabulary sizes and mask ids of LLaDA-8B (126,464 / 126,336), Dream
    (152,064 / 151,666) and DiffusionGemma (262,144, no mask id);
  * chunks of at most 4,096 tokens, documents of 296 tokens on average
    ("LLaDA-8B-MDLM-LoRA", Training table, row "Data");
  * a clean prefix plus an output canvas for the uniform-noise model
    ("diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes).
The datasets the pages train on (Nemotron-SFT-Code and others) are not used;
these synthetic draws stand in for them.

Typed-decision workloads (label slots of multiple-choice, score and yes/no
questions: "Native diffusion language-model training", Typed-decision
training and Labels) draw, from the CPU generator: a codebook of 128
distinct answer-token ids; per slot K ~ U[2, k_max] alternatives, answered by
the first K codebook tokens (every question spells its answers A, B, C, ...);
a label kind uniform over hard / dist / set with a uniform gold index, a
Dirichlet(1) distribution, or a uniform non-empty subset; then, on the
device generator, the slots' logits rows.

Draw order for a given seed (a fixed recipe, so a seed names one input):
  1. packed-document lengths (packed workloads only; CPU generator);
  2. clean ids;
  3. logits (diffusion / canvas), then encoder logits (uniform workloads),
     or hidden states then head weights (linear workloads; uniform linear
     workloads: canvas hidden states, encoder hidden states, head weights).
Normal draws are generated in fp32 in row blocks and rounded to bf16.
"N(0, s)" means standard deviation s.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch

ABSORBING, UNIFORM = 0, 1
ALIGNED, SHIFTED = 0, 1


@dataclass(frozen=True)
class Spec:
    key: str
    kind: str                  # "loss" | "linear"
    mode: int                  # ABSORBING | UNIFORM
    align: int                 # ALIGNED | SHIFTED
    vocab: int
    mask_id: int               # -1 when the noise has no mask token
    ids_high: int              # clean ids uniform in [0, ids_high]
    n_units: int = 1           # sequences (dense) -- packed: decided by lengths
    seq_len: int = 0           # dense sequence length (canvas length for uniform)
    prefix: int = 0            # uniform: clean prefix length before the canvas
    n_tokens_packed: int = 0   # packed: total tokens
    doc_mean: float = 296.0
    doc_min: int = 16
    doc_max: int = 4096
    std: float = 1.0           # logits std
    spike: float = 0.0         # added to the clean token's logit of each row
    d_model: int = 0
    h_std: float = 1.0
    w_std: float = 0.02
    eps: float = 1e-3
    enc_ar_weight: float = 0.0
    k_max: int = 0             # decision: alternatives per question in [2, k_max]
    data_seed: int = 0
    corrupt_seed: int = 0
    description: str = ""

    def scaled(self, **kw) -> "Spec":
        return replace(self, **kw)


WORKLOADS = {
    "abs_b2_l64_v1024": Spec(
        "abs_b2_l64_v1024", "loss", ABSORBING, ALIGNED, vocab=1024, mask_id=1023,
        ids_high=1022, n_units=2, seq_len=64, std=2.0, data_seed=0,
        description="tiny absorbing-mask loss, aligned logits, B=2 L=64 V=1024"),
    "abs_b1_l4096_v126464": Spec(
        "abs_b1_l4096_v126464", "loss", ABSORBING, ALIGNED, vocab=126464, mask_id=126336,
        ids_high=126335, n_units=1, seq_len=4096, std=3.0, spike=4.0, data_seed=2,
        description="LLaDA-like absorbing-mask loss, aligned logits, B=1 L=4096 V=126464, "
                    "clean-token logit +4"),
    "shift_b8_l2048_v152064": Spec(
        "shift_b8_l2048_v152064", "loss", ABSORBING, SHIFTED, vocab=152064, mask_id=151666,
        ids_high=151642, n_units=8, seq_len=2048, std=3.0, data_seed=3,
        description="Dream-like absorbing-mask loss, shifted logits, B=8 L=2048 V=152064"),
    "unif_b4_p512_c1024_v262144": Spec(
        "unif_b4_p512_c1024_v262144", "loss", UNIFORM, ALIGNED, vocab=262144, mask_id=-1,
        ids_high=262143, n_units=4, seq_len=1024, prefix=512, std=3.0, enc_ar_weight=1.0,
        data_seed=4,
        description="DiffusionGemma-like uniform-token noise, B=4, prefix 512 + canvas 1024, "
                    "V=262144, encoder AR weight 1"),
    "lin_t16384_d4096_v126464": Spec(
        "lin_t16384_d4096_v126464", "linear", ABSORBING, ALIGNED, vocab=126464,
        mask_id=126336, ids_high=126335, n_tokens_packed=16384, d_model=4096,
        h_std=1.0, w_std=0.02, data_seed=5,
        description="packed documents (lengths geometric, mean 296, 16..4096) through a fused "
                    "lm_head, T=16384 D=4096 V=126464"),
    # smaller cases of the same kernels, sized for detailed profiling (the
    # inputs are still larger than L2)
    "unif_b1_p256_c512_v262144": Spec(
        "unif_b1_p256_c512_v262144", "loss", UNIFORM, ALIGNED, vocab=262144, mask_id=-1,
        ids_high=262143, n_units=1, seq_len=512, prefix=256, std=3.0, enc_ar_weight=1.0,
        data_seed=6,
        description="DiffusionGemma-like uniform-token noise, B=1, prefix 256 + canvas 512, "
                    "V=262144 (every row scored; 0.67 GB of logits)"),
    "lin_unif_b4_p512_c1024_d4096_v262144": Spec(
        "lin_unif_b4_p512_c1024_d4096_v262144", "linear", UNIFORM, ALIGNED, vocab=262144,
        mask_id=-1, ids_high=262143, n_units=4, seq_len=1024, prefix=512, d_model=4096,
        h_std=1.0, w_std=0.02, enc_ar_weight=1.0, data_seed=7,
        description="DiffusionGemma-like uniform-token noise through a fused lm_head: B=4, "
                    "prefix 512 + canvas 1024, D=4096, V=262144, canvas and encoder hidden "
                    "states against one head, encoder AR weight 1"),
    "dec_s128_k26_v126464": Spec(
        "dec_s128_k26_v126464", "decision", ABSORBING, ALIGNED, vocab=126464, mask_id=126336,
        ids_high=126335, n_units=128, std=3.0, k_max=26, data_seed=8,
        description="typed-decision losses at 128 label slots (16 canvases x 8 questions), answer "
                    "tokens from a 26-letter codebook (K in [2, 26]), hard / dist / set labels, "
                    "logits at the label slots only, V=126464"),
    "lin_t4096_d4096_v32768": Spec(
        "lin_t4096_d4096_v32768", "linear", ABSORBING, ALIGNED, vocab=32768,
        mask_id=32767, ids_high=32000, n_tokens_packed=4096, d_model=4096,
        h_std=1.0, w_std=0.02, data_seed=5,
        description="packed documents through a fused lm_head, T=4096 D=4096 V=32768"),
}


def doc_lengths(total: int, mean: float, lo: int, hi: int, gen: torch.Generator) -> list:
    """Document lengths ~ Geometric(mean), clamped to [lo, hi], drawn until
    they cover `total`; the last document is cut to fit, and a remainder
    shorter than `lo` is merged into the previous document."""
    out = []
    acc = 0
    while acc < total:
        x = int(torch.empty(1, dtype=torch.float64).geometric_(1.0 / mean, generator=gen).item())
        x = max(lo, min(hi, x))
        out.append(x)
        acc += x
    over = acc - total
    out[-1] -= over
    if out[-1] < lo and len(out) > 1:
        out[-2] += out[-1]
        out.pop()
    return out


def _normal_bf16(rows: int, cols: int, std: float, gen: torch.Generator, device,
                 block_rows: int = 2048) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, block_rows):
        r1 = min(rows, r0 + block_rows)
        x = torch.randn((r1 - r0, cols), generator=gen, device=device, dtype=torch.float32)
        out[r0:r1] = (x * std).to(torch.bfloat16)
    return out


@dataclass
class Case:
    spec: Spec
    n_units: int
    seq_len: int                       # dense length (canvas length for uniform)
    cu_seqlens: Optional[torch.Tensor]  # int32 [n_units+1] or None
    pad_mask: Optional[torch.Tensor]    # uint8 or None
    clean: torch.Tensor                 # int32 [n_tokens] (canvas ids for uniform)
    logits: Optional[torch.Tensor] = None       # bf16 [rows, V]
    enc_clean: Optional[torch.Tensor] = None    # int32 [n_units*(prefix+seq_len)]
    enc_logits: Optional[torch.Tensor] = None   # bf16
    hidden: Optional[torch.Tensor] = None       # bf16 [T, D] (canvas rows for uniform)
    weight: Optional[torch.Tensor] = None       # bf16 [V, D]
    enc_hidden: Optional[torch.Tensor] = None   # bf16 [n_units*(prefix+seq_len), D]
    extra: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        return int(self.clean.shape[0])


def make_case(spec: Spec, device="cpu", seed: Optional[int] = None,
              with_tensors: bool = True) -> Case:
    """Draw one input of workload `spec` on `device` (torch generator of that
    device, seeded with `seed` or spec.data_seed)."""
    seed = spec.data_seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    cpu_gen = torch.Generator()
    cpu_gen.manual_seed(seed)

    if spec.kind == "decision":
        return _decision_case(spec, dev, gen, cpu_gen, with_tensors)

    if spec.kind == "linear" and spec.mode == UNIFORM:
        B, C, P = spec.n_units, spec.seq_len, spec.prefix
        full = torch.randint(0, spec.ids_high + 1, (B, P + C), generator=gen, device=dev,
                             dtype=torch.int64).to(torch.int32)
        canvas = full[:, P:].contiguous().reshape(-1)
        case = Case(spec, B, C, None, None, canvas, enc_clean=full.reshape(-1).contiguous())
        if with_tensors:
            case.hidden = _normal_bf16(B * C, spec.d_model, spec.h_std, gen, dev)
            case.enc_hidden = _normal_bf16(B * (P + C), spec.d_model, spec.h_std, gen, dev)
            case.weight = _normal_bf16(spec.vocab, spec.d_model, spec.w_std, gen, dev)
        return case

    if spec.kind == "linear":
        lens = doc_lengths(spec.n_tokens_packed, spec.doc_mean, spec.doc_min, spec.doc_max, cpu_gen)
        cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
        T = int(cu[-1])
        clean = torch.randint(0, spec.ids_high + 1, (T,), generator=gen, device=dev,
                              dtype=torch.int64).to(torch.int32)
        case = Case(spec, len(lens), 0, cu.to(dev), None, clean)
        if with_tensors:
            case.hidden = _normal_bf16(T, spec.d_model, spec.h_std, gen, dev)
            case.weight = _normal_bf16(spec.vocab, spec.d_model, spec.w_std, gen, dev)
        return case

    if spec.mode == UNIFORM:
        B, C, P = spec.n_units, spec.seq_len, spec.prefix
        full = torch.randint(0, spec.ids_high + 1, (B, P + C), generator=gen, device=dev,
                             dtype=torch.int64).to(torch.int32)
        canvas = full[:, P:].contiguous().reshape(-1)
        case = Case(spec, B, C, None, None, canvas, enc_clean=full.reshape(-1).contiguous())
        if with_tensors:
            case.logits = _normal_bf16(B * C, spec.vocab, spec.std, gen, dev)
            case.enc_logits = _normal_bf16(B * (P + C), spec.vocab, spec.std, gen, dev)
        return case

    B, L = spec.n_units, spec.seq_len
    clean = torch.randint(0, spec.ids_high + 1, (B * L,), generator=gen, device=dev,
                          dtype=torch.int64).to(torch.int32)
    case = Case(spec, B, L, None, None, clean)
    if with_tensors:
        if spec.spike != 0.0:
            logits = torch.empty((B * L, spec.vocab), dtype=torch.bfloat16, device=dev)
            block = 2048
            for r0 in range(0, B * L, block):
                r1 = min(B * L, r0 + block)
                x = torch.randn((r1 - r0, spec.vocab), generator=gen, device=dev,
                                dtype=torch.float32) * spec.std
                idx = clean[r0:r1].to(torch.int64)
                x[torch.arange(r1 - r0, device=dev), idx] += spec.spike
                logits[r0:r1] = x.to(torch.bfloat16)
            case.logits = logits
        else:
            case.logits = _normal_bf16(B * L, spec.vocab, spec.std, gen, dev)
    return case


HARD, DIST, SET = 0, 1, 2       # label kinds


def _decision_case(spec: Spec, dev, gen, cpu_gen, with_tensors: bool) -> Case:
    n = spec.n_units
    codebook = torch.randperm(spec.ids_high + 1, generator=cpu_gen)[:128].to(torch.int32)
    K = torch.randint(2, spec.k_max + 1, (n,), generator=cpu_gen)
    kind = torch.randint(0, 3, (n,), generator=cpu_gen).to(torch.int32)
    off = torch.zeros(n + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(K, 0).to(torch.int32)
    ids, vals = [], []
    for i in range(n):
        k = int(K[i])
        ids.append(codebook[:k])
        v = torch.zeros(k, dtype=torch.float32)
        if kind[i] == HARD:
            v[int(torch.randint(0, k, (1,), generator=cpu_gen))] = 1.0
        elif kind[i] == DIST:
            e = torch.empty(k, dtype=torch.float64).exponential_(generator=cpu_gen)
            v = (e / e.sum()).to(torch.float32)
        else:
            m = int(torch.randint(1, k + 1, (1,), generator=cpu_gen))
            v[torch.randperm(k, generator=cpu_gen)[:m]] = 1.0
        vals.append(v)
    case = Case(spec, n, 0, None, None, torch.zeros(n, dtype=torch.int32, device=dev))
    case.extra.update(cand_off=off.to(dev), cand_ids=torch.cat(ids).to(dev), kind=kind.to(dev),
                      val=torch.cat(vals).to(dev))
    if with_tensors:
        case.logits = _normal_bf16(n, spec.vocab, spec.std, gen, dev)
    return case


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
