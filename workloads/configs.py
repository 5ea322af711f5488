"""The synthetic decode workloads that parity tests and the benchmark run.

Shapes follow the long-context decode settings of "HHR: Hierarchical Hash
Retrieval for Efficient LLM Generation" (arXiv 2610.01230): Llama-3.1-8B /
Qwen3-style attention (32 query heads, 8 KV heads, head dim 128; Appendix A,
Table 3), 128-bit codes as the default hash length (Appendix A and C, "Hash Bit
Length"), 16-token pages, and contexts up to 128K (§4.3 "Context Length").
The budgets (pages kept P, tokens kept k) are fixed per workload.

Nothing here computes any part of the method; these are sizes and the recipe
for the seeded inputs (see ``workloads.synth``).
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    B: int            # sequences
    Hq: int           # query heads
    Hkv: int          # key/value heads
    d: int            # head dim
    N: int            # context length (valid keys) at the first decode step
    page: int         # page size S
    P: int            # pages kept per (sequence, KV head)
    k: int            # tokens kept per (sequence, KV head)
    bits: int         # code length b
    planted: int      # planted high-logit keys per (sequence, KV head)
    n_outlier: int    # outlier key channels per (sequence, KV head)
    outlier_scale: float
    rope_base: float = 0.0   # 0: no RoPE; else rotate-half RoPE with this base
    appends: int = 0         # decode steps with one appended key each
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def r(self) -> int:
        return self.Hq // self.Hkv

    @property
    def units(self) -> int:
        return self.B * self.Hkv

    @property
    def n_cap(self) -> int:
        return self.N + self.appends

    @property
    def words(self) -> int:
        return self.bits // 32

    def n_pages(self, n_valid: int | None = None) -> int:
        n = self.N if n_valid is None else n_valid
        return (n + self.page - 1) // self.page

    @property
    def np_cap(self) -> int:
        return (self.n_cap + self.page - 1) // self.page


_SEED0 = 0x48485200

WORKLOADS = {
    "tiny_4k": Workload(
        name="tiny_4k", B=1, Hq=1, Hkv=1, d=128, N=4096, page=16, P=32, k=128,
        bits=128, planted=16, n_outlier=4, outlier_scale=8.0, seed=_SEED0 + 0,
        notes="single head, 4K context"),
    "llama8b_32k": Workload(
        name="llama8b_32k", B=1, Hq=32, Hkv=8, d=128, N=32768, page=16, P=256,
        k=2048, bits=128, planted=64, n_outlier=4, outlier_scale=8.0,
        seed=_SEED0 + 1, notes="Llama-3.1-8B-shaped one-layer decode at 32K"),
    "llama8b_128k": Workload(
        name="llama8b_128k", B=1, Hq=32, Hkv=8, d=128, N=131072, page=16, P=512,
        k=4096, bits=128, planted=64, n_outlier=4, outlier_scale=8.0,
        seed=_SEED0 + 2, notes="Llama-3.1-8B-shaped one-layer decode at 128K"),
    "batch8_64k_b256": Workload(
        name="batch8_64k_b256", B=8, Hq=32, Hkv=8, d=128, N=65536, page=32, P=128,
        k=2048, bits=256, planted=64, n_outlier=round(0.05 * 128),
        outlier_scale=10.0, seed=_SEED0 + 3,
        notes="batched long-context decode, 256-bit codes, 32-token pages"),
    "llama8b_128k_paper": Workload(
        name="llama8b_128k_paper", B=1, Hq=32, Hkv=8, d=128, N=131072, page=16, P=2458,
        k=1966, bits=128, planted=64, n_outlier=4, outlier_scale=8.0,
        seed=_SEED0 + 2,
        notes="the 128K inputs with the paper's ratios: candidate budget 30% of the "
              "pages, Top-K 1.5% of the keys (Appendix A; §4.1)"),
    "qwen8b_128k_rope": Workload(
        name="qwen8b_128k_rope", B=4, Hq=32, Hkv=8, d=128, N=131072, page=16,
        P=512, k=4096, bits=128, planted=128, n_outlier=4, outlier_scale=8.0,
        rope_base=1.0e6, appends=16, seed=_SEED0 + 4,
        notes="Qwen3-8B-shaped prefill encode + 16 decode steps with appends"),
}

# Order used by tests and docs: the tiny case first, the headline case third.
ORDER = ["tiny_4k", "llama8b_32k", "llama8b_128k", "batch8_64k_b256", "qwen8b_128k_rope",
         "llama8b_128k_paper"]

HEADLINE = "llama8b_128k"


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    from dataclasses import replace
    return replace(w, **changes)
