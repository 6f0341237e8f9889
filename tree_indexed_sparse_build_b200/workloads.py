"""Named workload shapes for tree-indexed sparse decode attention.

Each entry fixes the cache shape, tree geometry (branching b, leaf block),
beam width and the synthetic-value recipe drawn by ``synth``.  Only shapes
and recipe parameters live here; no arithmetic of the method.

Tree geometry per workload (n0 = ceil(N / leaf_block) leaves, L = smallest
L >= 1 with b^L >= n0 scored levels below the single root):

=============  ======  ====  ==========  =======  ====  ==
name           N       b     leaf_block  n0       L     B
=============  ======  ====  ==========  =======  ====  ==
tiny_fp32      1024    2     16          64       6     2
gqa_32k        32768   8     64          512      3     8
decode_128k    131072  16    32          4096     3     16
deep_1m        1M      8     4           262144   6     8
build_256k     262144  4     16          16384    7     4
=============  ======  ====  ==========  =======  ====  ==
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    kv_heads: int
    q_heads: int
    head_dim: int
    seq_len: int
    kv_dtype: str            # "f32" or "bf16": storage of K, V and Q
    branching: int
    leaf_block: int
    beam: int
    nq: int = 1              # decode queries per query head per call
    needles: int = 0         # planted keys per KV head
    needle_amp: float = 0.0  # needle = amp * q_hat + N(0, sigma^2)
    needle_sigma: float = 0.0
    drift: bool = False      # low-rank positional drift added to K
    decode_steps: int = 0    # steps of {append 1 token, route, attend}
    append_tokens: int = 0   # tokens appended in one call after the build
    out_dtype: str = "bf16"
    seed: int = 0x2A000

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def units(self) -> int:
        return self.batch * self.kv_heads

    @property
    def scale(self) -> float:
        return self.head_dim ** -0.5

    @property
    def capacity(self) -> int:
        return self.seq_len + self.decode_steps + self.append_tokens

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    "tiny_fp32": Workload(
        name="tiny_fp32", batch=1, kv_heads=1, q_heads=1, head_dim=64, seq_len=1024,
        kv_dtype="f32", branching=2, leaf_block=16, beam=2, nq=16, needles=4,
        needle_amp=3.0, needle_sigma=0.1, out_dtype="f32", seed=0x2A000),
    "gqa_32k": Workload(
        name="gqa_32k", batch=8, kv_heads=8, q_heads=32, head_dim=128, seq_len=32768,
        kv_dtype="bf16", branching=8, leaf_block=64, beam=8, nq=1, needles=16,
        needle_amp=4.0, needle_sigma=0.2, seed=0x2A001),
    "decode_128k": Workload(
        name="decode_128k", batch=4, kv_heads=8, q_heads=32, head_dim=128, seq_len=131072,
        kv_dtype="bf16", branching=16, leaf_block=32, beam=16, nq=1, drift=True,
        decode_steps=64, seed=0x2A002),
    "deep_1m": Workload(
        name="deep_1m", batch=1, kv_heads=8, q_heads=64, head_dim=128, seq_len=1048576,
        kv_dtype="bf16", branching=8, leaf_block=4, beam=8, nq=1, needles=64,
        needle_amp=4.0, needle_sigma=0.2, seed=0x2A003),
    "build_256k": Workload(
        name="build_256k", batch=1, kv_heads=8, q_heads=32, head_dim=128, seq_len=262144,
        kv_dtype="bf16", branching=4, leaf_block=16, beam=4, nq=64, append_tokens=4096,
        seed=0x2A004),
}

# The 1M cache read with many independent queries in flight (64 per head).
THROUGHPUT_NQ = 64


def get(name: str) -> Workload:
    return WORKLOADS[name]
