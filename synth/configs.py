"""The five workloads of the hashed N-gram embedding layer, with their sub-table sizes.

Sub-table order is s = (n - 2) * K + (k - 1) for n = 2..N, k = 1..K.

Sub-table vocab sizes V_{n,k} follow the collision rule of "Scaling Embeddings
Outperforms Scaling Experts in Language Models" (section 3.2.2, Fig. 3b): a size near
an integer multiple of V0 makes 2-gram collisions spike, prime or not. So each
size is taken as the first distinct primes at or above floor((m + 1/2) * V0),
half-way between two multiples. The tiny config keeps its stated sizes
(4099/5003/6007/7001), which are fine for parity though close to multiples.
"""
from __future__ import annotations

from dataclasses import dataclass, field


def is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def primes_from(start: int, count: int) -> list:
    out, x = [], start
    while len(out) < count:
        if is_prime(x):
            out.append(x)
        x += 1
    return out


def mid_multiple_primes(V0: int, m: int, count: int) -> list:
    return primes_from((2 * m + 1) * V0 // 2, count)


@dataclass(frozen=True)
class NgramConfig:
    name: str
    V0: int
    D: int
    N: int
    K: int
    V_nk: tuple
    dtype: str                 # "bf16" or "f32"
    e_std: float = 0.02        # std of E_0 and every E_{n,k}
    seed: int = 0
    # workload shape
    num_seqs: int = 1
    seq_len: int = 0           # uniform length (0 = varlen)
    token_dist: str = "zipf"   # "zipf" or "uniform"
    zipf_alpha: float = 1.1
    decode_steps: int = 0      # >0: speculative decode workload
    tokens_per_step: int = 5   # 1 target token + 4 draft tokens
    prompt_max: int = 16       # decode: seeded prompt of 0..prompt_max ids per sequence
    extras: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def S(self) -> int:
        return (self.N - 1) * self.K

    @property
    def d(self) -> int:
        return self.D // self.S if self.S else 0

    @property
    def w_std(self) -> float:
        # "W ~ N(0, 1/16)" at width 16 is read as variance 1/width: std = width^-1/2.
        return self.d ** -0.5 if self.S else 0.0

    @property
    def ring_capacity(self) -> int:
        """Smallest power of two >= (N - 1) + tokens_per_step."""
        need = (self.N - 1) + self.tokens_per_step
        c = 1
        while c < need:
            c *= 2
        return c

    @property
    def elt_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def table_bytes(self) -> int:
        return sum(self.V_nk) * self.d * self.elt_bytes

    def with_(self, **kw) -> "NgramConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return NgramConfig(**d)


V0_BIG = 131072

TINY = NgramConfig(
    name="tiny_f32_D64_N3_K2", V0=1000, D=64, N=3, K=2, V_nk=(4099, 5003, 6007, 7001),
    dtype="f32", num_seqs=2, seq_len=64, token_dist="uniform")

PREFILL_D2048 = NgramConfig(
    name="prefill_bf16_D2048_N3_K2", V0=V0_BIG, D=2048, N=3, K=2,
    V_nk=tuple(mid_multiple_primes(V0_BIG, 16, 4)), dtype="bf16", num_seqs=8, seq_len=4096)

PREFILL_D4096_VARLEN = NgramConfig(
    name="prefill_varlen_bf16_D4096_N5_K2", V0=V0_BIG, D=4096, N=5, K=2,
    V_nk=tuple(mid_multiple_primes(V0_BIG, 25, 8)), dtype="bf16", num_seqs=16, seq_len=0,
    extras={"total_tokens": 65536, "len_lo": 256, "len_hi": 7936})

SPEC_DECODE = NgramConfig(
    name="spec_decode_bf16_D4096_N3_K4", V0=V0_BIG, D=4096, N=3, K=4,
    V_nk=tuple(mid_multiple_primes(V0_BIG, 25, 8)), dtype="bf16", num_seqs=256, seq_len=0,
    decode_steps=1000)

FULL_SCALE = NgramConfig(
    name="full_scale_bf16_D4096_N5_K2", V0=V0_BIG, D=4096, N=5, K=2,
    V_nk=tuple(mid_multiple_primes(V0_BIG, 55, 8)), dtype="bf16", num_seqs=8, seq_len=4096,
    decode_steps=1000, extras={"decode_seqs": 256})

# The decode half of the full-scale workload: the same layer and tables, 256 sequences x 5
# ids per step through a ring of the last N - 1 = 4 ids (capacity 16).
FULL_SCALE_DECODE = FULL_SCALE.with_(name="full_scale_decode_bf16_D4096_N5_K2", num_seqs=256, seq_len=0)

CONFIGS = [TINY, PREFILL_D2048, PREFILL_D4096_VARLEN, SPEC_DECODE, FULL_SCALE]
BY_NAME = {c.name: c for c in CONFIGS + [FULL_SCALE_DECODE]}


def same_tables(a: NgramConfig, b: NgramConfig) -> bool:
    """True when two workloads draw identical tables (same seed, shapes and value scales)."""
    return (a.seed, a.V0, a.D, a.V_nk, a.dtype, a.e_std, a.d, a.S > 0) == \
        (b.seed, b.V0, b.D, b.V_nk, b.dtype, b.e_std, b.d, b.S > 0)
