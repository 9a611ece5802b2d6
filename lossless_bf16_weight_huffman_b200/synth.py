"""Seeded synthetic BF16 weight sets (inputs only; none of the codec lives here).

Both the oracle's tests and the GPU path's tests and benchmark take their
inputs from this module, so the two sides see identical bits. Bulk generation
runs in ``csrc/synth.c`` (counter-based SplitMix64, Box-Muller normals,
round-to-nearest-even to BF16), threaded on the host cores.

Five weight sets, named by what they are:

* ``single_1024x4096``   one 1024x4096 tensor, N(0, 0.02).
* ``llama_layer``        one Llama-style decoder layer: q/o 4096x4096,
  k/v 1024x4096, gate/up 14336x4096, down 4096x14336, each
  N(0, 1/sqrt(fan_in)) with fan_in the second (input) dimension, plus two
  RMSNorm vectors of 4096 drawn as 1 + N(0, 0.02).
* ``heavy_tail_64m``     67,108,864 weights: 0.02 * Student-t(3), 0.1 % of
  them multiplied by 100, 1 % exact zeros (half +0, half -0), and at seeded
  distinct positions 64 subnormals, 8 +Inf, 8 -Inf and 16 NaNs (quiet and
  signalling payloads, both signs).
* ``llama8b_shaped``     32 layers of the decoder-layer shapes plus a
  128256x4096 embedding and a 128256x4096 lm_head, both N(0, 0.02).
* ``mixed_2000``         2000 tensors with sizes round(2^U(0,20)); each a
  bias N(0, 0.01), a norm vector 1 + N(0, 0.02), a 3x3 conv kernel
  N(0, 1/sqrt(9*C_in)) or a small linear N(0, 1/sqrt(fan_in)); tensor 0 has a
  single exponent (values in [1,2), random signs and fractions) and tensor 1
  (65,536 weights) cycles through all 256 exponents with equal counts.

Seeds: weight set k (1..5 in the order above) uses 0xDF110000 + k; tensor i of
a set uses splitmix64(set_seed, i).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libdfsynth.so")
_SRC = os.path.join(_HERE, "csrc", "synth.c")

NORMAL, STUDENT_T3, CONST_EXP, ALL_EXP = 0, 1, 2, 3

SET_NAMES = ("single_1024x4096", "llama_layer", "heavy_tail_64m", "llama8b_shaped", "mixed_2000")

_lib = None


def build_synth(force: bool = False) -> str:
    """Compile the generator library with gcc (host code, no GPU needed)."""
    import subprocess

    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build_synth()
        lib = ctypes.CDLL(_SO)
        lib.synth_splitmix64.restype = ctypes.c_uint64
        lib.synth_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_uniform.restype = ctypes.c_double
        lib.synth_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_f32_to_bf16_rne.restype = ctypes.c_uint16
        lib.synth_f32_to_bf16_rne.argtypes = [ctypes.c_float]
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_fill.argtypes = [
            ctypes.c_int, ctypes.c_uint64, ctypes.c_double, ctypes.c_double, ctypes.c_double,
            ctypes.c_double, ctypes.c_double, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int,
        ]
        _lib = lib
    return _lib


def splitmix64(seed: int, k: int) -> int:
    return int(_load().synth_splitmix64(seed & (2**64 - 1), k & (2**64 - 1)))


def uniform(seed: int, k: int) -> float:
    return float(_load().synth_uniform(seed & (2**64 - 1), k & (2**64 - 1)))


def set_seed(k: int) -> int:
    return 0xDF110000 + k


def _threads() -> int:
    return max(1, min(os.cpu_count() or 1, 64))


@dataclass
class TensorSpec:
    name: str
    shape: tuple
    kind: int
    seed: int
    mean: float = 0.0
    std: float = 0.0
    outlier_p: float = 0.0
    outlier_mul: float = 1.0
    zero_p: float = 0.0
    specials: bool = False  # heavy-tail set: subnormals, +-Inf, NaNs at seeded positions
    meta: dict = field(default_factory=dict)

    @property
    def numel(self) -> int:
        return int(math.prod(self.shape)) if self.shape else 1


def fill_ptr(spec: TensorSpec, ptr: int, n: int | None = None) -> None:
    """Generate ``spec`` into host memory at address ``ptr`` (n uint16 values)."""
    n = spec.numel if n is None else n
    rc = _load().synth_fill(
        spec.kind, spec.seed, spec.mean, spec.std, spec.outlier_p, spec.outlier_mul, spec.zero_p,
        ctypes.c_void_p(ptr), n, _threads(),
    )
    if rc != 0:
        raise ValueError(f"synth_fill failed for kind {spec.kind}")
    if spec.specials:
        arr = (ctypes.c_uint16 * n).from_address(ptr)
        view = np.frombuffer(arr, dtype=np.uint16)
        for pos, val in special_values(spec.seed, n):
            view[pos] = val


def generate(spec: TensorSpec) -> np.ndarray:
    """Return ``spec`` as a flat uint16 array of BF16 bit patterns."""
    out = np.empty(spec.numel, dtype=np.uint16)
    if out.size:
        fill_ptr(spec, out.ctypes.data, out.size)
    return out


def special_values(seed: int, n: int):
    """Seeded distinct positions and bit patterns of the heavy-tail set's specials:
    64 subnormals (exponent 0, fraction != 0, both signs), 8 +Inf, 8 -Inf and
    16 NaNs (quiet and signalling fractions, both signs)."""
    if n == 0:
        return []
    s = splitmix64(seed, 0x5350454349414C) ^ 0x5350454349414C
    values = []
    k = 0
    for i in range(64):
        r = splitmix64(s, 1_000_000 + i)
        sign = (r & 1) << 15
        frac = 1 + ((r >> 1) % 127)
        values.append(sign | frac)
    values += [0x7F80] * 8 + [0xFF80] * 8
    for i in range(16):
        r = splitmix64(s, 2_000_000 + i)
        sign = (i & 1) << 15
        if i & 2:  # quiet: top fraction bit set
            frac = 0x40 | ((r >> 2) & 0x3F)
        else:  # signalling: top fraction bit clear, fraction non-zero
            frac = 1 + ((r >> 2) % 63)
        values.append(sign | 0x7F80 | frac)
    want = min(len(values), n)
    positions = []
    seen = set()
    while len(positions) < want:
        p = splitmix64(s, k) % n
        k += 1
        if p not in seen:
            seen.add(p)
            positions.append(p)
    return list(zip(positions, values[:want]))


# --------------------------------------------------------------------------------------------
# weight sets


def single_1024x4096() -> list[TensorSpec]:
    return [TensorSpec("w", (1024, 4096), NORMAL, splitmix64(set_seed(1), 0), 0.0, 0.02)]


LAYER_SHAPES = (
    ("q_proj", (4096, 4096)),
    ("k_proj", (1024, 4096)),
    ("v_proj", (1024, 4096)),
    ("o_proj", (4096, 4096)),
    ("gate_proj", (14336, 4096)),
    ("up_proj", (14336, 4096)),
    ("down_proj", (4096, 14336)),
    ("input_layernorm", (4096,)),
    ("post_attention_layernorm", (4096,)),
)


def _layer(seed_base: int, first_index: int, prefix: str) -> list[TensorSpec]:
    out = []
    for j, (name, shape) in enumerate(LAYER_SHAPES):
        seed = splitmix64(seed_base, first_index + j)
        if len(shape) == 1:
            out.append(TensorSpec(prefix + name, shape, NORMAL, seed, 1.0, 0.02))
        else:
            out.append(TensorSpec(prefix + name, shape, NORMAL, seed, 0.0, 1.0 / math.sqrt(shape[1])))
    return out


def llama_layer() -> list[TensorSpec]:
    return _layer(set_seed(2), 0, "layers.0.")


def heavy_tail_64m() -> list[TensorSpec]:
    return [
        TensorSpec("w", (67108864,), STUDENT_T3, splitmix64(set_seed(3), 0), 0.0, 0.02,
                   outlier_p=0.001, outlier_mul=100.0, zero_p=0.01, specials=True)
    ]


VOCAB, HIDDEN, N_LAYERS = 128256, 4096, 32


def llama8b_shaped() -> list[TensorSpec]:
    base = set_seed(4)
    specs = [TensorSpec("embed_tokens", (VOCAB, HIDDEN), NORMAL, splitmix64(base, 0), 0.0, 0.02)]
    for layer in range(N_LAYERS):
        specs += _layer(base, 1 + layer * len(LAYER_SHAPES), f"layers.{layer}.")
    specs.append(TensorSpec("lm_head", (VOCAB, HIDDEN), NORMAL, splitmix64(base, 10_000), 0.0, 0.02))
    return specs


def mixed_2000(count: int = 2000) -> list[TensorSpec]:
    base = set_seed(5)
    draw = splitmix64(base, 0xD1CE)
    specs = []
    for i in range(count):
        seed = splitmix64(base, i)
        size = int(round(2.0 ** (20.0 * uniform(draw, 2 * i))))
        kind = min(3, int(4.0 * uniform(draw, 2 * i + 1)))
        if i == 0:
            specs.append(TensorSpec("t0.const_exponent", (size,), CONST_EXP, seed))
            continue
        if i == 1:
            specs.append(TensorSpec("t1.all_exponents", (65536,), ALL_EXP, seed))
            continue
        if kind == 0:
            specs.append(TensorSpec(f"t{i}.bias", (size,), NORMAL, seed, 0.0, 0.01))
        elif kind == 1:
            specs.append(TensorSpec(f"t{i}.norm", (size,), NORMAL, seed, 1.0, 0.02))
        elif kind == 2:
            c_in = max(1, int(math.sqrt(size / 9.0)))
            specs.append(TensorSpec(f"t{i}.conv3x3", (size,), NORMAL, seed, 0.0, 1.0 / math.sqrt(9.0 * c_in),
                                    meta={"c_in": c_in}))
        else:
            fan_in = max(1, int(math.sqrt(size)))
            specs.append(TensorSpec(f"t{i}.linear", (size,), NORMAL, seed, 0.0, 1.0 / math.sqrt(fan_in),
                                    meta={"fan_in": fan_in}))
    return specs


def weight_set(name: str) -> list[TensorSpec]:
    return {
        "single_1024x4096": single_1024x4096,
        "llama_layer": llama_layer,
        "heavy_tail_64m": heavy_tail_64m,
        "llama8b_shaped": llama8b_shaped,
        "mixed_2000": mixed_2000,
    }[name]()


def all_bf16_patterns() -> np.ndarray:
    """Every one of the 65,536 BF16 bit patterns, in order."""
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)
