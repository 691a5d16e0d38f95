"""Seeded synthetic inputs and the layer shapes of the pages' workloads.

Shared by the tests, ``bench.py`` and ``__graft_entry__``.  Holds none of the
method's arithmetic (no quantization, packing or product): only random draws and
shape tables.

Distributions (the pages measure on trained Llama / OPT weights; synthetic
draws of the same shapes stand in for them):

* x: ``randn(M, K)`` float32, rounded to bf16 (torch's RNE cast).
* W: ``0.02 * randn(N, K)`` float32 with outliers: an independent
  Bernoulli(0.001) mask from the same generator multiplies 0.1 % of the entries
  by 10.

Shapes (K, N) with W stored [N, K]:

* Llama-2-7B linears (gpt-fast pages): qkv (4096, 12288), o (4096, 4096),
  gate_up (4096, 22016), down (11008, 4096).
* Llama-70B linears (FP6-LLM / TC-FPx article, Llama linear layers): qkv
  (8192, 10240), o (8192, 8192), gate_up (8192, 57344), down (28672, 8192).
* OPT-30B linears (same article, OPT linear layers): qkv (7168, 21504),
  o (7168, 7168), fc1 (7168, 28672), fc2 (28672, 7168).
"""

import torch

LLAMA2_7B = {
    "qkv": (4096, 12288),
    "o": (4096, 4096),
    "gate_up": (4096, 22016),
    "down": (11008, 4096),
}
LLAMA_70B = {
    "qkv": (8192, 10240),
    "o": (8192, 8192),
    "gate_up": (8192, 57344),
    "down": (28672, 8192),
}
OPT_30B = {
    "qkv": (7168, 21504),
    "o": (7168, 7168),
    "fc1": (7168, 28672),
    "fc2": (28672, 7168),
}
SHAPE_SETS = {"llama2-7b": LLAMA2_7B, "llama-70b": LLAMA_70B, "opt-30b": OPT_30B}

OUTLIER_P = 0.001
OUTLIER_MUL = 10.0
W_STD = 0.02


def generator(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def activations(M, K, seed):
    """x bf16 [M, K] on the CPU: randn rounded to bf16."""
    g = generator(seed)
    return torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)


def weights(N, K, seed, rows=None):
    """W float32 [N, K] on the CPU: 0.02 * randn with 0.1 % of entries times 10.

    ``rows`` (optional slice) returns only those rows, drawn exactly as in the
    full matrix (row blocks are drawn with per-block generators so any block can
    be regenerated on its own).
    """
    return _weights_rows(N, K, seed, 0 if rows is None else rows.start, N if rows is None else rows.stop)


_BLOCK = 1024  # rows per independently seeded block


def _weights_rows(N, K, seed, r0, r1):
    out = torch.empty(max(r1 - r0, 0), K, dtype=torch.float32)
    b0 = r0 // _BLOCK
    b1 = (r1 + _BLOCK - 1) // _BLOCK
    for b in range(b0, b1):
        lo = b * _BLOCK
        hi = min(lo + _BLOCK, N)
        g = generator(seed * 1_000_003 + b)
        w = torch.randn(hi - lo, K, generator=g, dtype=torch.float32) * W_STD
        mask = torch.rand(hi - lo, K, generator=g) < OUTLIER_P
        w = torch.where(mask, w * OUTLIER_MUL, w)
        s0 = max(r0, lo)
        s1 = min(r1, hi)
        if s1 > s0:
            out[s0 - r0:s1 - r0] = w[s0 - lo:s1 - lo]
    return out


def integer_activations(M, K, seed, lo=-8, hi=8):
    """x bf16 [M, K] with small integer values (exact in bf16)."""
    g = generator(seed)
    return torch.randint(lo, hi + 1, (M, K), generator=g).to(torch.bfloat16)


def random_codes(shape, lo, hi, seed):
    """Uniform integer codes in [lo, hi] (inclusive), int64, for layout tests."""
    g = generator(seed)
    return torch.randint(lo, hi + 1, shape, generator=g)
