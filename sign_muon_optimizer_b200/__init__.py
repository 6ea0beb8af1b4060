"""Python binding of libsignmuon.so (the C ABI in include/signmuon.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels.  Device buffers are passed as torch CUDA tensors (or raw integer
device addresses); host buffers as numpy arrays.  The functions keep the C
names; each raises SignMuonError on a non-zero status.

The library must be built first (``python sign_muon_optimizer_b200/build.py``);
importing this package without it raises ImportError -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsignmuon.so")

# status codes, scales and flags (include/signmuon.h)
SIGNMUON_OK = 0
SIGNMUON_E_INVALID = 1
SIGNMUON_E_OVERFLOW = 2
SIGNMUON_E_NONFINITE = 3
SIGNMUON_E_CUDA = 4
SIGNMUON_E_NOMEM = 5
SIGNMUON_E_TIMEOUT = 6
SIGNMUON_E_UNSUPPORTED = 7
SIGNMUON_SCALE_FRO = 0
SIGNMUON_SCALE_SPECTRAL = 1
SIGNMUON_NS_FP32 = 1 << 0
SIGNMUON_NS_QUINTIC = 1 << 1
SIGNMUON_POST_POLAR = 1 << 2
SIGNMUON_ACC_INT8 = 1 << 3
SIGNMUON_ASYNC = 1 << 4
SIGNMUON_VOTE_ONLY = 1 << 5
SIGNMUON_KEEP_POLAR = 1 << 6
SIGNMUON_TIE_PLUS = 1 << 7
SIGNMUON_POLAR_AFTER_ONLY = 1 << 8
SIGNMUON_MUON_MEAN = 1 << 9
SIGNMUON_TERNARY = 1 << 10
SIGNMUON_NORMALIZED_SIGN = 1 << 11
SIGNMUON_PI_WARM = 1 << 12
SIGNMUON_NS_GRAM = 1 << 13

EXPORTED = [
    "signmuon_init", "signmuon_step", "signmuon_step_host", "signmuon_vote", "signmuon_pack",
    "signmuon_apply_update", "signmuon_polar", "signmuon_get_momentum", "signmuon_set_momentum",
    "signmuon_get_polar", "signmuon_get_signs", "signmuon_get_direction", "signmuon_get_scales",
    "signmuon_set_ns_coeffs", "signmuon_sync", "signmuon_info", "signmuon_plan",
    "signmuon_kernel_launches", "signmuon_last_error", "signmuon_status_string", "signmuon_destroy",
    "signmuon_profile", "signmuon_profile_read", "signmuon_get_gram",
    "signmuon_spectral_norm_noalloc", "signmuon_sign_ternary", "signmuon_vote_ternary",
    "signmuon_get_ternary_signs", "signmuon_local_signs", "signmuon_vote_step", "signmuon_sums_step",
    "signmuon_plan_tables", "signmuon_get_pi_state", "signmuon_set_pi_state", "signmuon_vote_step_ptrs",
    "signmuon_ipc_get_handle", "signmuon_ipc_open", "signmuon_ipc_close",
]
PROF_KINDS = ["momentum", "norm_finalize", "ns_gram", "ns_square", "ns_apply", "power_iter", "pack",
              "vote", "stage", "post_gram", "post_square", "post_apply", "update", "k0_scale"]


class SignMuonError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"signmuon status {status}: {msg}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python sign_muon_optimizer_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_uint
    PP = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "signmuon_init": (I, [ctypes.POINTER(P), ctypes.POINTER(I64), I, I, F, F, I, F, I, I, U, P]),
        "signmuon_step": (I, [P, P, PP, F]),
        "signmuon_step_host": (I, [P, P, PP, F]),
        "signmuon_vote": (I, [P, PP, I64, P, P]),
        "signmuon_pack": (I, [P, P, I64, P]),
        "signmuon_sign_ternary": (I, [P, P, I64, P]),
        "signmuon_vote_ternary": (I, [P, PP, I64, P, P]),
        "signmuon_get_ternary_signs": (I, [P, I, P]),
        "signmuon_get_pi_state": (I, [P, I, P]),
        "signmuon_set_pi_state": (I, [P, I, P]),
        "signmuon_local_signs": (I, [P, P, PP, P, I64]),
        "signmuon_vote_step": (I, [P, P, P, I64, I, F]),
        "signmuon_vote_step_ptrs": (I, [P, P, PP, I, F]),
        "signmuon_ipc_get_handle": (I, [P, P, ctypes.POINTER(I64)]),
        "signmuon_ipc_open": (I, [P, ctypes.POINTER(P)]),
        "signmuon_ipc_close": (I, [P]),
        "signmuon_sums_step": (I, [P, P, P, F]),
        "signmuon_plan_tables": (I, [ctypes.POINTER(I64), I, I, I, I, I, U, ctypes.c_char_p, I64,
                                     ctypes.POINTER(I64)]),
        "signmuon_apply_update": (I, [P, P, P, I64, F]),
        "signmuon_polar": (I, [P, PP, PP]),
        "signmuon_get_momentum": (I, [P, I, P]),
        "signmuon_set_momentum": (I, [P, I, P]),
        "signmuon_get_polar": (I, [P, I, P]),
        "signmuon_get_signs": (I, [P, I, P]),
        "signmuon_get_direction": (I, [P, P]),
        "signmuon_get_scales": (I, [P, P]),
        "signmuon_set_ns_coeffs": (I, [P, ctypes.POINTER(F), I]),
        "signmuon_sync": (I, [P]),
        "signmuon_info": (I, [P, ctypes.POINTER(I64), I]),
        "signmuon_plan": (I, [ctypes.POINTER(I64), I, I, I, I, I, U, ctypes.POINTER(I64), I]),
        "signmuon_kernel_launches": (I64, []),
        "signmuon_last_error": (ctypes.c_char_p, [P]),
        "signmuon_status_string": (ctypes.c_char_p, [I]),
        "signmuon_destroy": (None, [P]),
        "signmuon_profile": (I, [P, I]),
        "signmuon_get_gram": (I, [P, I, I, P]),
        "signmuon_spectral_norm_noalloc": (I, [P, I64, I64, I, P, P]),
        "signmuon_profile_read": (I, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64), I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _ptr(x):
    """Device/host address of a torch tensor, numpy array or int."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _ptr_array(xs):
    arr = (ctypes.c_void_p * len(xs))()
    for i, x in enumerate(xs):
        arr[i] = _ptr(x)
    return arr


def _check(h, rc):
    if rc != 0:
        raise SignMuonError(rc, _lib.signmuon_last_error(h).decode(errors="replace"))


def _shapes_arr(shapes):
    flat = [int(v) for rc in shapes for v in rc]
    return (ctypes.c_int64 * max(1, len(flat)))(*flat), len(shapes)


def _default_stream():
    try:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
    except Exception:
        pass
    return None


# ---- functions with the C names -------------------------------------------

def signmuon_init(shapes, M, beta, lam, K, eps, scale, P=1, flags=0, stream=None):
    if isinstance(scale, str):
        scale = {"fro": SIGNMUON_SCALE_FRO, "spectral": SIGNMUON_SCALE_SPECTRAL}[scale]
    arr, n = _shapes_arr(shapes)
    h = ctypes.c_void_p()
    if stream is None:
        stream = _default_stream()
    rc = _lib.signmuon_init(ctypes.byref(h), arr, n, int(M), float(beta), float(lam), int(K), float(eps),
                            int(scale), int(P), int(flags), stream)
    _check(None, rc)
    return h


def signmuon_step(h, W, G, eta):
    _check(h, _lib.signmuon_step(h, _ptr(W), _ptr_array(G), float(eta)))


def signmuon_step_host(h, W_host, G_host, eta):
    _check(h, _lib.signmuon_step_host(h, _ptr(W_host), _ptr_array(G_host), float(eta)))


def signmuon_vote(h, signs, d, sums=None, majority=None):
    _check(h, _lib.signmuon_vote(h, _ptr_array(signs), int(d), _ptr(sums), _ptr(majority)))


def signmuon_pack(h, U, d, out):
    _check(h, _lib.signmuon_pack(h, _ptr(U), int(d), _ptr(out)))


def signmuon_sign_ternary(h, U, d, out):
    _check(h, _lib.signmuon_sign_ternary(h, _ptr(U), int(d), _ptr(out)))


def signmuon_vote_ternary(h, signs, d, sums=None, majority=None):
    _check(h, _lib.signmuon_vote_ternary(h, _ptr_array(signs), int(d), _ptr(sums), _ptr(majority)))


def signmuon_get_ternary_signs(h, m, dst):
    _check(h, _lib.signmuon_get_ternary_signs(h, int(m), _ptr(dst)))


def signmuon_local_signs(h, W, G, signs, stride):
    _check(h, _lib.signmuon_local_signs(h, _ptr(W), _ptr_array(G), _ptr(signs), int(stride)))


def signmuon_vote_step(h, W, signs, stride, M, eta):
    _check(h, _lib.signmuon_vote_step(h, _ptr(W), _ptr(signs), int(stride), int(M), float(eta)))


def signmuon_vote_step_ptrs(h, W, signs, eta):
    """signs: one device pointer (int or tensor) per worker, in worker order."""
    _check(h, _lib.signmuon_vote_step_ptrs(h, _ptr(W), _ptr_array(signs), len(signs), float(eta)))


SIGNMUON_IPC_HANDLE_BYTES = 64


def signmuon_ipc_get_handle(dev_ptr):
    """(handle bytes, byte offset of dev_ptr in its allocation)."""
    buf = ctypes.create_string_buffer(SIGNMUON_IPC_HANDLE_BYTES)
    off = ctypes.c_int64()
    _check(None, _lib.signmuon_ipc_get_handle(_ptr(dev_ptr), buf, ctypes.byref(off)))
    return buf.raw, int(off.value)


def signmuon_ipc_open(handle):
    """Base address, in this process, of a peer's allocation."""
    if len(handle) != SIGNMUON_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has 64 bytes")
    base = ctypes.c_void_p()
    _check(None, _lib.signmuon_ipc_open(ctypes.create_string_buffer(bytes(handle), SIGNMUON_IPC_HANDLE_BYTES),
                                        ctypes.byref(base)))
    return int(base.value)


def signmuon_ipc_close(base):
    _check(None, _lib.signmuon_ipc_close(_ptr(base)))


def signmuon_sums_step(h, W, sums, eta):
    _check(h, _lib.signmuon_sums_step(h, _ptr(W), _ptr(sums), float(eta)))


def signmuon_apply_update(h, W, D, d, eta):
    _check(h, _lib.signmuon_apply_update(h, _ptr(W), _ptr(D), int(d), float(eta)))


def signmuon_polar(h, X, U):
    _check(h, _lib.signmuon_polar(h, _ptr_array(X), _ptr_array(U)))


def signmuon_get_momentum(h, m, dst):
    _check(h, _lib.signmuon_get_momentum(h, int(m), _ptr(dst)))


def signmuon_set_momentum(h, m, src):
    _check(h, _lib.signmuon_set_momentum(h, int(m), _ptr(src)))


def signmuon_get_pi_state(h, which, dst):
    _check(h, _lib.signmuon_get_pi_state(h, int(which), _ptr(dst)))


def signmuon_set_pi_state(h, which, src):
    _check(h, _lib.signmuon_set_pi_state(h, int(which), _ptr(src)))


def signmuon_get_polar(h, m, dst):
    _check(h, _lib.signmuon_get_polar(h, int(m), _ptr(dst)))


def signmuon_get_signs(h, m, dst):
    _check(h, _lib.signmuon_get_signs(h, int(m), _ptr(dst)))


def signmuon_get_direction(h, dst):
    _check(h, _lib.signmuon_get_direction(h, _ptr(dst)))


def signmuon_get_scales(h, M, n_mats):
    out = np.zeros(M * n_mats, np.float32)
    _check(h, _lib.signmuon_get_scales(h, out.ctypes.data))
    return out.reshape(M, n_mats)


def signmuon_spectral_norm_noalloc(X, rows, cols, P, sigma, stream=None):
    """Power-iteration sigma of one matrix without any device allocation
    (see include/signmuon.h); X and sigma are device buffers."""
    if stream is None:
        stream = _default_stream()
    _check(None, _lib.signmuon_spectral_norm_noalloc(_ptr(X), int(rows), int(cols), int(P), _ptr(sigma), stream))


def signmuon_get_gram(h, m, mat, g):
    out = np.zeros((g, g), np.float32)
    _check(h, _lib.signmuon_get_gram(h, int(m), int(mat), out.ctypes.data))
    return out


def signmuon_set_ns_coeffs(h, coeffs):
    c = (ctypes.c_float * len(coeffs))(*[float(v) for v in coeffs])
    _check(h, _lib.signmuon_set_ns_coeffs(h, c, len(coeffs)))


def signmuon_sync(h):
    _check(h, _lib.signmuon_sync(h))


INFO_KEYS = ["d", "packed_bytes", "device_bytes", "groups", "M", "n_mats", "pi_state_workers", "pi_state_single"]


def signmuon_info(h):
    out = (ctypes.c_int64 * 8)()
    _check(h, _lib.signmuon_info(h, out, 8))
    return dict(zip(INFO_KEYS, list(out)))


def signmuon_plan(shapes, M, K=5, scale=SIGNMUON_SCALE_FRO, P=1, flags=0):
    if isinstance(scale, str):
        scale = {"fro": SIGNMUON_SCALE_FRO, "spectral": SIGNMUON_SCALE_SPECTRAL}[scale]
    arr, n = _shapes_arr(shapes)
    out = (ctypes.c_int64 * 8)()
    _check(None, _lib.signmuon_plan(arr, n, int(M), int(K), int(scale), int(P), int(flags), out, 8))
    return dict(zip(INFO_KEYS, list(out)))


def signmuon_plan_tables(shapes, M, K=5, scale=SIGNMUON_SCALE_FRO, P=1, flags=0):
    """The plan's tables (host only) as a dict parsed from the library's JSON."""
    import json
    if isinstance(scale, str):
        scale = {"fro": SIGNMUON_SCALE_FRO, "spectral": SIGNMUON_SCALE_SPECTRAL}[scale]
    arr, n = _shapes_arr(shapes)
    need = ctypes.c_int64(0)
    args = (arr, n, int(M), int(K), int(scale), int(P), int(flags))
    _check(None, _lib.signmuon_plan_tables(*args, None, 0, ctypes.byref(need)))
    buf = ctypes.create_string_buffer(need.value)
    _check(None, _lib.signmuon_plan_tables(*args, buf, need.value, ctypes.byref(need)))
    return json.loads(buf.value.decode())


def signmuon_kernel_launches():
    return int(_lib.signmuon_kernel_launches())


def signmuon_last_error(h=None):
    return _lib.signmuon_last_error(h).decode(errors="replace")


def signmuon_status_string(status):
    return _lib.signmuon_status_string(int(status)).decode()


def signmuon_destroy(h):
    _lib.signmuon_destroy(h)


def signmuon_profile(h, enable):
    _check(h, _lib.signmuon_profile(h, 1 if enable else 0))


def signmuon_profile_read(h):
    """{kind: (total ms, launches)} since the last read (waits for the stream)."""
    n = len(PROF_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(h, _lib.signmuon_profile_read(h, ms, cnt, n))
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(PROF_KINDS)}


class SignMuon:
    """Owning wrapper of a handle: ``SignMuon(shapes, M, ...)`` then
    ``.step(W, G, eta)``; the remaining methods mirror the C calls."""

    def __init__(self, shapes, M, beta=0.9, lam=0.01, K=5, eps=1e-7, scale="fro", P=1, flags=0,
                 stream=None):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.M = int(M)
        self.flags = int(flags)
        # the CUDA stream the handle enqueues on (a cudaStream_t as an int; 0
        # or None for the legacy default stream)
        self.stream = stream if stream is not None else _default_stream()
        self.h = signmuon_init(self.shapes, M, beta, lam, K, eps, scale, P, flags, self.stream)
        self.info = signmuon_info(self.h)
        self.d = self.info["d"]

    def step(self, W, G, eta):
        signmuon_step(self.h, W, G, eta)

    def step_host(self, W, G, eta):
        signmuon_step_host(self.h, W, G, eta)

    def vote(self, signs, d, sums=None, majority=None):
        signmuon_vote(self.h, signs, d, sums, majority)

    def pack(self, U, d, out):
        signmuon_pack(self.h, U, d, out)

    def sign_ternary(self, U, d, out):
        signmuon_sign_ternary(self.h, U, d, out)

    def vote_ternary(self, signs, d, sums=None, majority=None):
        signmuon_vote_ternary(self.h, signs, d, sums, majority)

    def get_ternary_signs(self, m, dst):
        signmuon_get_ternary_signs(self.h, m, dst)

    def sign_stride(self):
        """Bytes per worker in a sign buffer for local_signs / vote_step: the
        packed bits (or, with SIGNMUON_TERNARY, the int8 signs) rounded up to
        16."""
        n = self.d if self.flags & SIGNMUON_TERNARY else (self.d + 7) // 8
        return (n + 15) // 16 * 16

    def local_signs(self, W, G, signs, stride=None):
        signmuon_local_signs(self.h, W, G, signs, self.sign_stride() if stride is None else stride)

    def vote_step(self, W, signs, M, eta, stride=None):
        signmuon_vote_step(self.h, W, signs, self.sign_stride() if stride is None else stride, M, eta)

    def vote_step_ptrs(self, W, signs, eta):
        signmuon_vote_step_ptrs(self.h, W, signs, eta)

    def sums_step(self, W, sums, eta):
        signmuon_sums_step(self.h, W, sums, eta)

    def apply_update(self, W, D, d, eta):
        signmuon_apply_update(self.h, W, D, d, eta)

    def polar(self, X, U):
        signmuon_polar(self.h, X, U)

    def get_momentum(self, m, dst):
        signmuon_get_momentum(self.h, m, dst)

    def set_momentum(self, m, src):
        signmuon_set_momentum(self.h, m, src)

    def get_polar(self, m, dst):
        signmuon_get_polar(self.h, m, dst)

    def get_pi_state(self, which, dst):
        signmuon_get_pi_state(self.h, which, dst)

    def set_pi_state(self, which, src):
        signmuon_set_pi_state(self.h, which, src)

    def get_signs(self, m, dst):
        signmuon_get_signs(self.h, m, dst)

    def get_direction(self, dst):
        signmuon_get_direction(self.h, dst)

    def get_gram(self, m, mat):
        r, c = self.shapes[mat]
        return signmuon_get_gram(self.h, m, mat, min(r, c))

    def get_scales(self):
        return signmuon_get_scales(self.h, self.M, len(self.shapes))

    def set_ns_coeffs(self, coeffs):
        signmuon_set_ns_coeffs(self.h, coeffs)

    def sync(self):
        signmuon_sync(self.h)

    def profile(self, enable=True):
        signmuon_profile(self.h, enable)

    def profile_read(self):
        return signmuon_profile_read(self.h)

    def close(self):
        if self.h is not None:
            signmuon_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
