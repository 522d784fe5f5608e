"""Seeded synthetic inputs shared by the oracle and the CUDA path.

Holds no arithmetic of the method: it draws numbers (Philox-4x32-10, and
normals by inversion through a 65 536-cell quantile table; see synth.c), rounds
them to the stored formats, and writes expert blobs in the runtime layout.  The
C source is compiled on first use.
"""
import ctypes
import os
import subprocess
import threading

import numpy as np

from .configs import AR_PHI, AR_SIG, CONFIGS, MoeConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

W_CODE = {"f32": 0, "bf16": 1, "int4": 2, "nvfp4": 3}
T_TOKENS, T_AR1, T_ROUTER = 8, 9, 4


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, -O3)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-mavx2", "-mfma", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            u64, i32, f32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
            L.synth_normal_f32.argtypes = [u64, i32, i32, i32, u64, u64, f32, vp]
            L.synth_round_bf16.argtypes = [vp, u64, vp]
            L.synth_quantise_int4.argtypes = [vp, i32, i32, vp, vp]
            L.synth_quantise_nvfp4_rows.argtypes = [vp, i32, i32, f32, vp, vp]
            L.synth_blob_bytes.argtypes = [i32, i32, i32]
            L.synth_blob_bytes.restype = u64
            L.synth_expert_blob.argtypes = [u64, i32, i32, i32, i32, i32, i32, f32, vp]
            L.synth_fill_pool.argtypes = [u64, i32, i32, i32, i32, i32, f32, vp, u64, i32]
            L.synth_ar1.argtypes = [u64, i32, i32, i32, f32, f32, vp]
            L.synth_philox4x32_10.argtypes = [vp, vp, vp]
            L.synth_normal_f32_scalar.argtypes = [u64, i32, i32, i32, u64, u64, f32, vp]
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_f32(seed, tensor, layer, expert, n, sigma=1.0, offset=0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_f32(seed, tensor, layer, expert, offset, n, sigma, _ptr(out))
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    """The bare Philox-4x32-10 bijection of the generator (4 counter words, 2 key words)."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    assert c.shape == (4,) and k.shape == (2,)
    out = np.empty(4, dtype=np.uint32)
    lib().synth_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def normal_f32_scalar(seed, tensor, layer, expert, n, sigma=1.0, offset=0) -> np.ndarray:
    """normal_f32 through the scalar one-block path (for checking the vectorised path)."""
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_f32_scalar(seed, tensor, layer, expert, offset, n, sigma, _ptr(out))
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().synth_round_bf16(_ptr(a), a.size, _ptr(out))
    return out


def quantise_int4(w: np.ndarray):
    """int4 g128 quantiser (data preparation): returns (packed uint8 [R, K/2], bf16 scale bits [R, K/128])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, K = w.shape
    assert K % 128 == 0
    q = np.empty((R, K // 2), dtype=np.uint8)
    s = np.empty((R, K // 128), dtype=np.uint16)
    lib().synth_quantise_int4(_ptr(w), R, K, _ptr(q), _ptr(s))
    return q, s


def quantise_nvfp4(w: np.ndarray, g: float):
    """nvfp4 quantiser for rows of w with global scale g: (packed e2m1 [R, K/2], e4m3 codes [R, K/16])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, K = w.shape
    assert K % 16 == 0
    q = np.empty((R, K // 2), dtype=np.uint8)
    s = np.empty((R, K // 16), dtype=np.uint8)
    lib().synth_quantise_nvfp4_rows(_ptr(w), R, K, g, _ptr(q), _ptr(s))
    return q, s


def expert_weights_f32(cfg: MoeConfig, layer: int, expert: int, shared: bool = False):
    """The N(0, sigma) draws behind one expert blob, before rounding / quantisation."""
    tg, tu, td = (5, 6, 7) if shared else (1, 2, 3)
    ex = 0 if shared else expert
    H, I = cfg.H, cfg.I
    wg = normal_f32(cfg.seed, tg, layer, ex, I * H, cfg.sigma).reshape(I, H)
    wu = normal_f32(cfg.seed, tu, layer, ex, I * H, cfg.sigma).reshape(I, H)
    wd = normal_f32(cfg.seed, td, layer, ex, H * I, cfg.sigma).reshape(H, I)
    return wg, wu, wd


def expert_blob(cfg: MoeConfig, layer: int, expert: int, shared: bool = False, out=None) -> np.ndarray:
    if out is None:
        out = np.empty(cfg.blob_bytes, dtype=np.uint8)
    rc = lib().synth_expert_blob(cfg.seed, layer, expert, int(shared), cfg.H, cfg.I,
                                 W_CODE[cfg.wdtype], cfg.sigma, _ptr(out))
    if rc:
        raise RuntimeError("synth_expert_blob failed: %d" % rc)
    return out


def fill_pool(cfg: MoeConfig, base_ptr: int, stride: int = None, nthreads: int = None) -> None:
    """Writes all L*E routed blobs at base_ptr + (l*E+e)*stride (host memory)."""
    stride = stride or cfg.blob_bytes
    nthreads = nthreads or os.cpu_count() or 1
    rc = lib().synth_fill_pool(cfg.seed, cfg.L, cfg.E, cfg.H, cfg.I, W_CODE[cfg.wdtype],
                               cfg.sigma, base_ptr, stride, nthreads)
    if rc:
        raise RuntimeError("synth_fill_pool failed: %d" % rc)


def router_weights(cfg: MoeConfig, layer: int) -> np.ndarray:
    """W_r [E, H] fp32, N(0, sigma)."""
    return normal_f32(cfg.seed, T_ROUTER, layer, 0, cfg.E * cfg.H, cfg.sigma).reshape(cfg.E, cfg.H)


def ar1_chain(seed: int, chain: int, T: int, H: int) -> np.ndarray:
    out = np.empty((T, H), dtype=np.float32)
    lib().synth_ar1(seed, chain, T, H, AR_PHI, AR_SIG, _ptr(out))
    return out


def tokens(cfg: MoeConfig, batch: int):
    """Hidden states of the whole run as [steps, batch, H] float32.

    iid: N(0,1).  ar1: `batch` independent chains (chain b = key field b), each
    tokens/batch long; step s holds time s of every chain.  bf16 workloads round
    once to bf16 (RNE); the returned float32 values are then exactly those bf16s.
    Returns (values_f32, bf16_bits or None).
    """
    H = cfg.H
    steps = cfg.tokens // batch
    if cfg.process == "iid":
        x = normal_f32(cfg.seed, T_TOKENS, 0, 0, cfg.tokens * H, 1.0).reshape(steps, batch, H)
    else:
        chains = [ar1_chain(cfg.seed, b, steps, H) for b in range(batch)]
        x = np.stack(chains, axis=1)
    x = np.ascontiguousarray(x, dtype=np.float32)
    if cfg.x_dtype == "bf16":
        bits = round_bf16(x)
        vals = (bits.astype(np.uint32) << 16).view(np.float32)
        return vals, bits
    return x, None


__all__ = ["MoeConfig", "CONFIGS", "build", "lib", "normal_f32", "normal_f32_scalar", "philox4x32_10", "round_bf16",
           "quantise_int4", "quantise_nvfp4", "expert_weights_f32", "expert_blob", "fill_pool", "router_weights",
           "ar1_chain", "tokens"]
