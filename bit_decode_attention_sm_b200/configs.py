"""The five HeadQ decode workloads, with their sizes.

Each entry describes one synthetic decode layer shaped like the workloads of
"HeadQ: Model-Visible Distortion and Score-Space Correction for KV-Cache
Quantization" (gist.science technical summary, section 5: K-only decode with
dense values and a full-KV 2-bit composition).  The pages run on WikiText-103
activations of six models; none of that is available, so seeded synthetic
keys, values and queries of these shapes stand in for it.

Fields
------
B, Hq, Hkv, d, T : batch, query heads, KV heads, head dim, cached tokens.
r                : HeadQ side-code rank (columns of U_h).
r_s              : rank of the synthetic query structure (A in q = A g + 0.1 eps).
n_cal            : calibration queries per query head for the query-PCA basis.
kv_dtype         : "f32" or "bf16" for the keys/values fed to the cache write.
vmode            : "dense" (V stored as kv_dtype) or "2bit" (V quantised like
                   the base key code, no side code).
drift            : std of the per-channel random-walk step of the key means
                   along the position axis (0 = no drift).
prefill          : tokens per sequence written by one cache-write call when the
                   cache write itself is timed.
seed             : generator seed.
"""

from dataclasses import dataclass, asdict


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    r: int
    r_s: int
    n_cal: int
    kv_dtype: str
    vmode: str
    drift: float
    prefill: int
    seed: int

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def as_dict(self):
        return asdict(self)

    def with_(self, **kw) -> "Workload":
        d = asdict(self)
        d.update(kw)
        return Workload(**d)


WORKLOADS = (
    # Tiny single head, fp32 keys and values: 16 decode queries read one cache.
    Workload("tiny-1head-d64-T512-fp32", B=1, Hq=16, Hkv=1, d=64, T=512, r=8,
             r_s=8, n_cal=256, kv_dtype="f32", vmode="dense", drift=0.0,
             prefill=512, seed=0),
    # Small MHA decode layer.
    Workload("mha-12h-d64-B8-T2048", B=8, Hq=12, Hkv=12, d=64, T=2048, r=8,
             r_s=8, n_cal=256, kv_dtype="bf16", vmode="dense", drift=0.0,
             prefill=2048, seed=1),
    # GQA 7B-class layer, group 7.
    Workload("gqa-28q4kv-d128-B16-T8192", B=16, Hq=28, Hkv=4, d=128, T=8192,
             r=16, r_s=16, n_cal=1024, kv_dtype="bf16", vmode="dense",
             drift=0.0, prefill=8192, seed=2),
    # Long-context GQA layer, group 4, drifting key means: the bandwidth case.
    Workload("longctx-32q8kv-d128-B1-T131072", B=1, Hq=32, Hkv=8, d=128,
             T=131072, r=16, r_s=16, n_cal=1024, kv_dtype="bf16",
             vmode="dense", drift=0.01, prefill=131072, seed=3),
    # Full-KV 2-bit composition: HeadQ keys plus 2-bit values.
    Workload("fullkv2bit-28q4kv-d128-B64-T4096", B=64, Hq=28, Hkv=4, d=128,
             T=4096, r=16, r_s=16, n_cal=1024, kv_dtype="bf16", vmode="2bit",
             drift=0.0, prefill=4096, seed=4),
)


def workload(i_or_name) -> Workload:
    if isinstance(i_or_name, int):
        return WORKLOADS[i_or_name]
    for w in WORKLOADS:
        if w.name == i_or_name:
            return w
    raise KeyError(i_or_name)
