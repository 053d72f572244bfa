"""Seeded synthetic inputs for the MXFP4 routed-expert MoE layer.

This package draws numbers and lays out bytes; it contains none of the
layer's arithmetic.  The fp64 oracle (``oracle/``) and the CUDA library both
take their inputs from here.  The generator itself is C (``k3gen.c``, built
on first use with gcc + OpenMP) so the K3-shape expert blobs (896 x 17.5 MB)
can be produced quickly.

The workloads mirror the shapes the source pages give for Kimi K3's MoE layer
(896 routed experts, top-16, one always-on shared expert; "kimi-k3-in-c"
project card, core features: 17 bytes per 32 MXFP4 weights), with hidden and
FFN sizes d=7168, ff=1536.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "k3gen.c")
_LIB = os.path.join(_HERE, "libk3gen.so")
_lock = threading.Lock()
_lib = None

# Streams of the counter-based generator.
STREAM_X, STREAM_ROUTER, STREAM_BIAS, STREAM_NIB, STREAM_SCALE, STREAM_SHARED, STREAM_ZIPF, STREAM_NORM = range(8)

# E8M0 exponents of the synthetic experts: uniform in [118, 124].
SCALE_LO, SCALE_COUNT = 118, 7
# Standard deviation of the bf16 shared-expert weights.  0.16 is close to the
# rms (0.1596) of a routed expert's decoded weights under the distribution
# above, so the shared and routed terms have comparable size.
SHARED_SIGMA = 0.16


def build(force: bool = False) -> str:
    """Compile libk3gen.so next to its source (gcc, OpenMP)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(
                ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64, u32, i32, dbl = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_int32, ctypes.c_double)
        vp = ctypes.c_void_p
        lib.k3gen_base.argtypes = [u64, u64]
        lib.k3gen_base.restype = u64
        lib.k3gen_draw.argtypes = [u64, u64, u64]
        lib.k3gen_draw.restype = u64
        lib.k3gen_normal.argtypes = [u64, u64, u64]
        lib.k3gen_normal.restype = dbl
        lib.k3gen_bf16_bits.argtypes = [dbl]
        lib.k3gen_bf16_bits.restype = ctypes.c_uint16
        lib.k3gen_normal_bf16.argtypes = [u64, u64, u64, u64, dbl, vp]
        lib.k3gen_normal_bf16.restype = None
        lib.k3gen_normal_f32.argtypes = [u64, u64, u64, u64, dbl, vp]
        lib.k3gen_normal_f32.restype = None
        lib.k3gen_uniform_bytes.argtypes = [u64, u64, u64, u64, vp]
        lib.k3gen_uniform_bytes.restype = None
        lib.k3gen_uniform_range_u8.argtypes = [u64, u64, u64, u64, u32, u32, vp]
        lib.k3gen_uniform_range_u8.restype = None
        lib.k3gen_zipf_bias.argtypes = [u64, u64, i32, dbl, vp, vp]
        lib.k3gen_zipf_bias.restype = ctypes.c_int
        lib.k3gen_blob_bytes.argtypes = [i64, i64]
        lib.k3gen_blob_bytes.restype = u64
        lib.k3gen_expert_blob.argtypes = [u64, i64, i64, i64, u32, u32, vp]
        lib.k3gen_expert_blob.restype = None
        lib.k3gen_shared.argtypes = [u64, i64, i64, dbl, vp, vp, vp]
        lib.k3gen_shared.restype = None
        _lib = lib
    return _lib


@dataclasses.dataclass(frozen=True)
class Config:
    """One MoE-layer workload.

    bias: None (no router bias), "normal" (b_e ~ N(0,1), stream 2) or
    "zipf" (b_e = -1.1 ln r_e for a seeded rank permutation, stream 6).
    out_fp32: the output mode the workload is quoted in (the parity tests
    check both modes on every config).
    scale_lo, scale_count: the experts' E8M0 bytes are uniform in
    [scale_lo, scale_lo + scale_count) (the workloads: 118..124).
    """
    name: str
    d: int
    ff: int
    E: int
    k: int
    ff_shared: int
    T: int
    bias: str | None = None
    zipf_s: float = 1.1
    out_fp32: bool = False
    scale_lo: int = SCALE_LO
    scale_count: int = SCALE_COUNT

    @property
    def blob_bytes(self) -> int:
        return blob_bytes(self.d, self.ff)


CONFIGS = {
    # d=256, ff=128, E=32, top-4, one bf16 shared expert, T=4
    "tiny": Config("tiny", d=256, ff=128, E=32, k=4, ff_shared=128, T=4),
    # K3 shape, single-token decode
    "k3_decode": Config("k3_decode", d=7168, ff=1536, E=896, k=16, ff_shared=1536, T=1),
    # K3 shape, 8-token decode, per-expert router bias ~ N(0,1)
    "k3_decode_t8": Config("k3_decode_t8", d=7168, ff=1536, E=896, k=16, ff_shared=1536, T=8,
                           bias="normal"),
    # K3 shape, 512-token prefill, Zipf(1.1)-skewed router prior
    "k3_prefill_512": Config("k3_prefill_512", d=7168, ff=1536, E=896, k=16, ff_shared=1536,
                             T=512, bias="zipf"),
    # K3 shape, 4096-token prefill, uniform routing, bf16 output
    "k3_prefill_4096": Config("k3_prefill_4096", d=7168, ff=1536, E=896, k=16,
                              ff_shared=1536, T=4096),
}


def blob_bytes(d: int, ff: int) -> int:
    """Bytes of one routed expert: 3 matrices of d*ff weights at 17 B per 32."""
    return 3 * d * ff * 17 // 32


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    """Standard normals number offset..offset+n-1 of a stream, fp64."""
    lib = _load()
    return np.array([lib.k3gen_normal(seed, stream, offset + i) for i in range(n)])


def bf16_bits(v: float) -> int:
    """Bits of the bfloat16 nearest (ties to even) to a double."""
    return int(_load().k3gen_bf16_bits(float(v)))


def hidden(cfg: Config, seed: int = 0, T: int | None = None) -> np.ndarray:
    """x: [T, d] bfloat16 bits (uint16), entries bf16(N(0,1)), stream 0."""
    T = cfg.T if T is None else T
    out = np.empty((T, cfg.d), dtype=np.uint16)
    _load().k3gen_normal_bf16(seed, STREAM_X, 0, out.size, 1.0, _ptr(out))
    return out


def router(cfg: Config, seed: int = 0) -> np.ndarray:
    """W_r: [E, d] fp32, entries fp32(N(0, 1/d)), stream 1."""
    out = np.empty((cfg.E, cfg.d), dtype=np.float32)
    _load().k3gen_normal_f32(seed, STREAM_ROUTER, 0, out.size, 1.0 / math.sqrt(cfg.d), _ptr(out))
    return out


def bias(cfg: Config, seed: int = 0) -> np.ndarray | None:
    """Router bias [E] fp32 or None."""
    if cfg.bias is None:
        return None
    out = np.empty((cfg.E,), dtype=np.float32)
    if cfg.bias == "normal":
        _load().k3gen_normal_f32(seed, STREAM_BIAS, 0, cfg.E, 1.0, _ptr(out))
    elif cfg.bias == "zipf":
        rc = _load().k3gen_zipf_bias(seed, STREAM_ZIPF, cfg.E, cfg.zipf_s, _ptr(out), None)
        if rc != 0:
            raise ValueError("zipf bias: E out of range")
    else:
        raise ValueError(cfg.bias)
    return out


def expert_blob(cfg: Config, e: int, seed: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """Routed expert e as one blob of uint8 (layout in k3gen.c)."""
    nb = cfg.blob_bytes
    if out is None:
        out = np.empty((nb,), dtype=np.uint8)
    assert out.dtype == np.uint8 and out.size == nb
    if not (0 <= cfg.scale_lo and cfg.scale_count >= 1 and cfg.scale_lo + cfg.scale_count <= 256):
        raise ValueError("E8M0 byte range outside 0..255")
    _load().k3gen_expert_blob(seed, e, cfg.d, cfg.ff, cfg.scale_lo, cfg.scale_count, _ptr(out))
    return out


def all_blobs(cfg: Config, seed: int = 0) -> np.ndarray:
    """All E blobs, [E, blob_bytes] uint8 (small configs only)."""
    out = np.empty((cfg.E, cfg.blob_bytes), dtype=np.uint8)
    for e in range(cfg.E):
        expert_blob(cfg, e, seed, out[e])
    return out


def norm_weights(cfg: Config, seed: int = 0) -> np.ndarray:
    """RMSNorm weights [d] as bf16 bits: bf16(1 + 0.1 N(0,1)), stream 7."""
    out = np.empty((cfg.d,), dtype=np.uint16)
    base = normal(seed, STREAM_NORM, 0, cfg.d)
    for j in range(cfg.d):
        out[j] = bf16_bits(1.0 + 0.1 * base[j])
    return out


def shared(cfg: Config, seed: int = 0):
    """Shared expert (W_g,s [ff_s,d], W_u,s [ff_s,d], W_d,s [d,ff_s]) as bf16 bits."""
    wg = np.empty((cfg.ff_shared, cfg.d), dtype=np.uint16)
    wu = np.empty((cfg.ff_shared, cfg.d), dtype=np.uint16)
    wd = np.empty((cfg.d, cfg.ff_shared), dtype=np.uint16)
    _load().k3gen_shared(seed, cfg.d, cfg.ff_shared, SHARED_SIGMA, _ptr(wg), _ptr(wu), _ptr(wd))
    return wg, wu, wd


def plane_offsets(d: int, ff: int):
    """Byte offsets of the six planes inside a blob, in blob order:
    (g_nib, g_scale, u_nib, u_scale, d_nib, d_scale)."""
    mat = d * ff
    offs = []
    o = 0
    for _ in range(3):
        offs.append(o)
        o += mat // 2
        offs.append(o)
        o += mat // 32
    return tuple(offs)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)
