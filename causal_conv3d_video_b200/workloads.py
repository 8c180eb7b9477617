"""Synthetic decoder-shaped workloads for the cached causal Conv3D.

Shapes only: no arithmetic of the operator lives here.  Every workload is a
single call signature (plus the seeded value recipe) in NTHWC layout, N=1.
The value recipe follows the decoder study's synthetic-latent practice
("Cache-Aware Conv3D Lowering Across Embedded World-Model Decoders", evaluation
setup of Tab. 2: decoder-compatible synthetic BF16 latents, batch size 1): activations
N(0,1), weights N(0, 1/(Cin*kt*kh*kw)) (variance), bias N(0, sigma_b^2).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Conv:
    name: str
    Cin: int
    Cout: int
    H: int
    W: int
    T_x: int
    cache_len: int
    N: int = 1
    kt: int = 3
    kh: int = 3
    kw: int = 3
    pad_t_base: int | None = None
    cache_keep: int | None = None
    stride: tuple = (1, 1)          # (s_h, s_w)
    pad: tuple = (1, 1)
    dilation: tuple = (1, 1, 1)
    dtype: str = "bf16"
    sigma_b: float = 0.02
    has_bias: bool = True
    seed: int = 0
    stride_t: int = 1               # temporal stride (> 1: encoder downsampling)

    def __post_init__(self):
        if self.pad_t_base is None:
            object.__setattr__(self, "pad_t_base", self.dilation[0] * (self.kt - 1))
        if self.cache_keep is None:
            object.__setattr__(self, "cache_keep", self.pad_t_base)

    def replace(self, **kw) -> "Conv":
        if "dilation" in kw or "kt" in kw:
            kw.setdefault("pad_t_base", None)
            kw.setdefault("cache_keep", None)
        return dataclasses.replace(self, **kw)

    # ---- derived sizes (plain shape formulas; used for reporting only) ----
    @property
    def out_hw(self):
        s_h, s_w = self.stride
        p_h, p_w = self.pad
        _, d_h, d_w = self.dilation
        H_o = (self.H + 2 * p_h - d_h * (self.kh - 1) - 1) // s_h + 1
        W_o = (self.W + 2 * p_w - d_w * (self.kw - 1) - 1) // s_w + 1
        return H_o, W_o

    def synth_kwargs(self):
        return dict(N=self.N, Cin=self.Cin, Cout=self.Cout, H=self.H, W=self.W,
                    T_x=self.T_x, cache_len=self.cache_len, kt=self.kt,
                    kh=self.kh, kw=self.kw, dtype=self.dtype, seed=self.seed,
                    sigma_b=self.sigma_b, has_bias=self.has_bias)


# -- the five workload families -------------------------------------------
# small fp32 case, 16 channels, 16x16, 2-frame cache + 3 frames
C1 = Conv("fp32_16ch_16x16_c2_t3", 16, 16, 16, 16, T_x=3, cache_len=2,
          dtype="fp32", sigma_b=0.1)
# decoder bottleneck, per-latent-frame chunk: 384 ch at 90x160
C2 = Conv("bf16_384ch_90x160_c2_t1", 384, 384, 90, 160, T_x=1, cache_len=2)
C2_EMPTY = C2.replace(name="bf16_384ch_90x160_c0_t1", cache_len=0)
# full-resolution decoder stage: 96 ch at 720x1280, 4 frames per chunk
C3 = Conv("bf16_96ch_720x1280_c2_t4", 96, 96, 720, 1280, T_x=4, cache_len=2,
          sigma_b=0.1)
C3B = C3.replace(name="bf16_192to96_720x1280_c2_t4", Cin=192)
# contract-edge sweep
C4_TIME = Conv("bf16_3x1x1_384to768_180x320_c2_t1", 384, 768, 180, 320, T_x=1,
               cache_len=2, kh=1, kw=1, pad=(0, 0))
C4_DIL = Conv("bf16_192ch_dt2_180x320_c4_t1", 192, 192, 180, 320, T_x=1,
              cache_len=4, dilation=(2, 1, 1))
C4_STRIDE = Conv("bf16_192ch_s2_360x640_c2_t1", 192, 192, 360, 640, T_x=1,
                 cache_len=2, stride=(2, 2))
C4_C1 = C2.replace(name="bf16_384ch_90x160_c1_t1", cache_len=1)
C4_ODD = Conv("bf16_192ch_89x157_c2_t1", 192, 192, 89, 157, T_x=1, cache_len=2)
# encoder-side temporal downsampling (stride 2 in time; the paper leaves these
# calls on native Conv3D): a 3x1x1 time conv and a 3x3x3 conv, 4-frame chunks
C6_ST2_TIME = Conv("bf16_3x1x1_384ch_st2_180x320_c2_t4", 384, 384, 180, 320, T_x=4,
                   cache_len=2, kh=1, kw=1, pad=(0, 0), stride_t=2)
C6_ST2 = Conv("bf16_192ch_st2_180x320_c2_t4", 192, 192, 180, 320, T_x=4, cache_len=2,
              stride_t=2)

# the decoder's RGB output conv (96 -> 3 channels at 720x1280, 4-frame chunks):
# too thin in Cout for the tensor-core tiles, it runs on the FFMA path
C_RGB = Conv("bf16_96to3_720x1280_c2_t4", 96, 3, 720, 1280, T_x=4, cache_len=2, sigma_b=0.1)

WORKLOADS = {c.name: c for c in (
    C1, C2, C2_EMPTY, C3, C3B, C4_TIME, C4_DIL, C4_STRIDE, C4_C1, C4_ODD, C6_ST2_TIME,
    C6_ST2, C_RGB)}
# cache-length sweep {0,1,2} on the bottleneck and on the stride-2 signature
for _base in (C2, C4_STRIDE):
    for _c in (0, 1, 2):
        _w = _base.replace(name=f"{_base.name.rsplit('_c', 1)[0]}_c{_c}_t{_base.T_x}",
                           cache_len=_c)
        WORKLOADS.setdefault(_w.name, _w)

BENCH_WORKLOAD = C2


# -- synthetic 17-frame decode schedule --------------------------------------
@dataclass(frozen=True)
class ModuleGroup:
    Cin: int
    Cout: int
    kernel: tuple
    H: int
    W: int
    count: int


# 5 latent frames -> 17 output frames; 16-ch latent at 90x160.
DECODE17_GROUPS = (
    ModuleGroup(16, 384, (3, 3, 3), 90, 160, 1),
    ModuleGroup(384, 384, (3, 3, 3), 90, 160, 6),
    ModuleGroup(384, 384, (3, 3, 3), 180, 320, 6),
    ModuleGroup(384, 768, (3, 1, 1), 180, 320, 3),
    ModuleGroup(384, 384, (3, 3, 3), 360, 640, 2),
    ModuleGroup(384, 768, (3, 1, 1), 360, 640, 3),
    ModuleGroup(384, 192, (3, 3, 3), 360, 640, 1),
    ModuleGroup(192, 192, (3, 3, 3), 360, 640, 4),
    ModuleGroup(192, 96, (3, 3, 3), 720, 1280, 1),
    ModuleGroup(96, 96, (3, 3, 3), 720, 1280, 7),
)
# frames per chunk at each spatial size (the first chunk carries one frame)
DECODE17_FRAMES = {(90, 160): (1, 1, 1, 1, 1), (180, 320): (1, 1, 1, 1, 1),
                   (360, 640): (1, 2, 2, 2, 2), (720, 1280): (1, 4, 4, 4, 4)}


@dataclass
class ScheduledCall:
    module: int
    group: int
    chunk: int
    conv: Conv


def decode17_schedule(scale_hw: tuple | None = None):
    """The 164-call sequence: per chunk, every module in order.

    3x3x3 modules run on all 5 chunks with |C| = min(frames seen, 2).
    3x1x1 (time-upsampling) modules skip chunk 0, whose frame only seeds their
    cache, and run on chunks 1-4.  ``scale_hw`` replaces every spatial size
    (same channels, caches and frames) for a cheap oracle-checkable copy.
    """
    calls, module = [], 0
    modules = []
    for g, grp in enumerate(DECODE17_GROUPS):
        for _ in range(grp.count):
            modules.append((module, g, grp))
            module += 1
    for chunk in range(5):
        for m, g, grp in modules:
            frames = DECODE17_FRAMES[(grp.H, grp.W)]
            kt, kh, kw = grp.kernel
            temporal_only = (kh == 1 and kw == 1)
            if temporal_only and chunk == 0:
                continue
            seen = sum(frames[:chunk])
            H, W = scale_hw if scale_hw else (grp.H, grp.W)
            conv = Conv(f"m{m}_g{g}_k{chunk}", grp.Cin, grp.Cout, H, W,
                        T_x=frames[chunk], cache_len=min(seen, 2), kt=kt, kh=kh,
                        kw=kw, pad=(0, 0) if temporal_only else (1, 1),
                        seed=1000 + 10 * m + chunk)
            calls.append(ScheduledCall(m, g, chunk, conv))
    return calls


def signature(c: Conv):
    return (c.Cin, c.Cout, c.kt, c.kh, c.kw, c.H, c.W, c.T_x, c.cache_len,
            c.stride, c.pad, c.dilation, c.dtype, c.stride_t)


def decode17_records(scale_hw: tuple | None = None):
    """The 164-call schedule as plain records (the content of
    configs/decode17.json): one dict per call, in call order."""
    out = []
    for c in decode17_schedule(scale_hw):
        v = c.conv
        out.append({"call": len(out), "module": c.module, "group": c.group, "chunk": c.chunk,
                    "Cin": v.Cin, "Cout": v.Cout, "kernel": [v.kt, v.kh, v.kw], "H": v.H,
                    "W": v.W, "T_x": v.T_x, "cache_len": v.cache_len,
                    "pad_t_base": v.pad_t_base, "cache_keep": v.cache_keep,
                    "stride": list(v.stride), "pad": list(v.pad),
                    "dilation": list(v.dilation), "dtype": v.dtype})
    return out
