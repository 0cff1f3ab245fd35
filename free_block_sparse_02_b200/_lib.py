"""ctypes binding of libsparsepr.so (the C ABI in include/sparsepr.h).

Argument marshalling only: every step of the operator runs in the library's CUDA kernels.
PyTorch provides device memory (the workspace and outputs) and the CUDA stream.  If the
library is missing the binding raises; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparsepr.so")

SPARSEPR_F32 = 0
SPARSEPR_BF16 = 1

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "workspace", 5: "numeric", 6: "timeout", 7: "call out of order"}

Q_KLABELS, Q_QLABELS, Q_ROUTE, Q_PROBES, Q_PROBE_W, Q_FIT, Q_KCENT, Q_QCENT, Q_OSP, Q_ODENSE, \
    Q_STATS, Q_KOBJ, Q_QOBJ, Q_KM_PATH = range(1, 15)
# kernels a pair of events can bracket (SPARSEPR_KERNEL_* in the C header)
KERNEL_BLOCK_SPARSE, KERNEL_KMEANS_ASSIGN, KERNEL_KMEANS_UPDATE, KERNEL_KMEANS_LOOP = range(4)


class SparsePRError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("s", ctypes.c_int32), ("n_kgroups", ctypes.c_int32),
                ("n_qgroups", ctypes.c_int32), ("density", ctypes.c_float), ("fixed_k", ctypes.c_int32),
                ("P", ctypes.c_int32), ("probe_mode", ctypes.c_int32), ("lambda_", ctypes.c_double),
                ("km_iters", ctypes.c_int32), ("km_iters_warm", ctypes.c_int32), ("km_tol", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("partition", ctypes.c_int32), ("repair", ctypes.c_int32),
                ("correction", ctypes.c_int32), ("trunc_rank", ctypes.c_int32), ("key_rank", ctypes.c_int32)]


class HeadStats(ctypes.Structure):
    _fields_ = [("k_iters", ctypes.c_int32), ("q_iters", ctypes.c_int32), ("k_refined", ctypes.c_int32),
                ("q_refined", ctypes.c_int32), ("fit_retries", ctypes.c_int32), ("span_rank", ctypes.c_int32),
                ("sparse_pairs", ctypes.c_int64), ("density", ctypes.c_double),
                ("k_objective", ctypes.c_double), ("q_objective", ctypes.c_double), ("lambda_", ctypes.c_double)]


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with free_block_sparse_02_b200.build.build()")
    lib = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    cfgp = ctypes.POINTER(Config)
    sig = {
        "sparsepr_workspace_size": (i32, [cfgp, ctypes.POINTER(sz)]),
        "sparsepr_plan_create": (i32, [cfgp, vp, sz, ctypes.POINTER(vp)]),
        "sparsepr_plan": (i32, [vp, vp, vp, vp]),
        "sparsepr_set_partition": (i32, [vp, vp, vp, vp, vp, vp, vp]),
        "sparsepr_attention": (i32, [vp, vp, vp, vp, vp]),
        "sparsepr_fit_apply": (i32, [vp, vp, i32, vp]),
        "sparsepr_plan_query": (i32, [vp, i32, vp, sz]),
        "sparsepr_sync": (i32, [vp]),
        "sparsepr_plan_destroy": (None, [vp]),
        "sparsepr_status_string": (ctypes.c_char_p, [i32]),
        "sparsepr_version": (i32, []),
        "sparsepr_set_kernel_events": (i32, [vp, i32, vp, vp]),
        "sparsepr_launch_count": (ctypes.c_int64, []),
        "sparsepr_set_wait_limit": (i32, [vp, i32, ctypes.c_int64]),
        "sparsepr_set_kmeans_path": (i32, [vp, i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise SparsePRError(status, where)


def config_from(w, **over) -> Config:
    """C config from a Workload (or any object with the same attribute names)."""
    g = lambda k: over.get(k, getattr(w, k))
    return Config(B=g("B"), H=g("H"), N=g("N"), d=g("d"), dtype=g("dtype"), s=g("s"),
                  n_kgroups=g("n_kgroups"), n_qgroups=g("n_qgroups"), density=g("density"),
                  fixed_k=g("fixed_k"), P=g("P"), probe_mode=g("probe_mode"), lambda_=g("lam"),
                  km_iters=g("km_iters"), km_iters_warm=g("km_iters_warm"), km_tol=g("km_tol"),
                  seed=g("seed"), partition=over.get("partition", getattr(w, "partition", 0)),
                  repair=over.get("repair", getattr(w, "repair", 1)),
                  correction=over.get("correction", getattr(w, "correction", 0)),
                  trunc_rank=over.get("trunc_rank", getattr(w, "trunc_rank", 0)),
                  key_rank=over.get("key_rank", getattr(w, "key_rank", 0)))


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(load().sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "sparsepr_workspace_size")
    return n.value


def launch_count() -> int:
    """Kernels launched by the library since it was loaded."""
    return int(load().sparsepr_launch_count())


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class SparsePR:
    """One plan object: a workspace on `device` plus the library's plan handle."""

    def __init__(self, w, device="cuda", **over):
        self.lib = load()
        self.cfg = config_from(w, **over)
        self.dtype = torch.float32 if self.cfg.dtype == SPARSEPR_F32 else torch.bfloat16
        self.shape = (self.cfg.B, self.cfg.H, self.cfg.N, self.cfg.d)
        self.ws_bytes = workspace_size(self.cfg)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        h = ctypes.c_void_p()
        _check(self.lib.sparsepr_plan_create(ctypes.byref(self.cfg), _ptr(self.workspace), self.ws_bytes,
                                             ctypes.byref(h)), "sparsepr_plan_create")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and getattr(self, "lib", None) is not None:
            self.lib.sparsepr_plan_destroy(h)
            self.handle = None

    def _chk(self, t: torch.Tensor, name: str):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == self.dtype and tuple(t.shape) == self.shape):
            raise ValueError(f"{name}: expected a contiguous CUDA {self.dtype} tensor of shape {self.shape}")

    def plan(self, Q, K, stream=None):
        self._chk(Q, "Q")
        self._chk(K, "K")
        _check(self.lib.sparsepr_plan(self.handle, _ptr(Q), _ptr(K), _stream(stream)), "sparsepr_plan")

    def set_partition(self, klabels, qlabels, route, probes, probe_w, stream=None):
        kl = np.ascontiguousarray(klabels, dtype=np.int32)
        ql = np.ascontiguousarray(qlabels, dtype=np.int32)
        rt = np.ascontiguousarray(route, dtype=np.uint8)
        pr = np.ascontiguousarray(probes, dtype=np.int32)
        pw = np.ascontiguousarray(probe_w, dtype=np.float64)
        BH, N, P = self.cfg.B * self.cfg.H, self.cfg.N, self.cfg.P
        if kl.size != BH * N or ql.size != BH * N or rt.size != BH * self.cfg.n_qgroups * self.cfg.n_kgroups \
                or pr.size != BH * P or pw.size != BH * P:
            raise ValueError("set_partition: array sizes do not match the configuration")
        c = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        _check(self.lib.sparsepr_set_partition(self.handle, c(kl), c(ql), c(rt), c(pr), c(pw), _stream(stream)),
               "sparsepr_set_partition")

    def attention(self, Q, K, V, stream=None):
        for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
            self._chk(t, n)
        _check(self.lib.sparsepr_attention(self.handle, _ptr(Q), _ptr(K), _ptr(V), _stream(stream)),
               "sparsepr_attention")

    def fit_apply(self, O=None, out_dtype=None, stream=None):
        if O is None:
            O = torch.empty(self.shape, dtype=out_dtype or self.dtype, device=self.workspace.device)
        if not (O.is_cuda and O.is_contiguous() and tuple(O.shape) == self.shape
                and O.dtype in (torch.float32, torch.bfloat16)):
            raise ValueError("O: expected a contiguous CUDA float32/bfloat16 tensor of the input shape")
        code = SPARSEPR_F32 if O.dtype == torch.float32 else SPARSEPR_BF16
        _check(self.lib.sparsepr_fit_apply(self.handle, _ptr(O), code, _stream(stream)), "sparsepr_fit_apply")
        return O

    def __call__(self, Q, K, V, O=None, out_dtype=None, stream=None):
        self.plan(Q, K, stream)
        self.attention(Q, K, V, stream)
        return self.fit_apply(O, out_dtype, stream)

    def set_kernel_events(self, start: "torch.cuda.Event", stop: "torch.cuda.Event", kernel: int = 0):
        """Bracket one kernel launch with two (already created) CUDA events: kernel 0 = the
        block-sparse attention, 1 = the first key k-means assignment, 2 = the first key k-means
        update, 3 = the whole key k-means loop when it runs in one launch (KERNEL_*)."""
        h0 = ctypes.c_void_p(start.cuda_event) if start is not None else None
        h1 = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
        _check(self.lib.sparsepr_set_kernel_events(self.handle, int(kernel), h0, h1), "sparsepr_set_kernel_events")

    def set_wait_limit(self, cycles: int, kernel: int = 0):
        """Test hook of the timeout path: the given kernel's bounded device-side waits give up
        after `cycles` SM cycles (0 restores the default of about 1 s)."""
        _check(self.lib.sparsepr_set_wait_limit(self.handle, int(kernel), int(cycles)), "sparsepr_set_wait_limit")

    def set_kmeans_path(self, mode: int):
        """Test hook of the k-means paths: 1 launches the steps of every Lloyd iteration
        separately even where the whole loop fits one launch; 0 restores the automatic choice."""
        _check(self.lib.sparsepr_set_kmeans_path(self.handle, int(mode)), "sparsepr_set_kmeans_path")

    def sync(self):
        _check(self.lib.sparsepr_sync(self.handle), "sparsepr_sync")

    # ---------------------------------------------------------------- results
    def query(self, what: int) -> np.ndarray:
        c = self.cfg
        BH = c.B * c.H
        spec = {
            Q_KLABELS: (np.int32, (BH, c.N)), Q_QLABELS: (np.int32, (BH, c.N)),
            Q_ROUTE: (np.uint8, (BH, c.n_qgroups, c.n_kgroups)), Q_PROBES: (np.int32, (BH, c.P)),
            Q_PROBE_W: (np.float64, (BH, c.P)), Q_FIT: (np.float64, (BH, c.d + 1, c.d)),
            Q_KCENT: (np.float64, (BH, c.n_kgroups, c.d)), Q_QCENT: (np.float64, (BH, c.n_qgroups, c.n_kgroups)),
            Q_OSP: (np.float32, (BH, c.N, c.d)), Q_ODENSE: (np.float32, (BH, c.P, c.d)),
            Q_KOBJ: (np.float64, (BH, c.km_iters)), Q_QOBJ: (np.float64, (BH, c.km_iters)),
            Q_KM_PATH: (np.int32, (2,)),
        }[what]
        out = np.empty(spec[1], dtype=spec[0])
        _check(self.lib.sparsepr_plan_query(self.handle, what, out.ctypes.data_as(ctypes.c_void_p), out.nbytes),
               "sparsepr_plan_query")
        return out

    def stats(self) -> List[Dict[str, float]]:
        BH = self.cfg.B * self.cfg.H
        arr = (HeadStats * BH)()
        _check(self.lib.sparsepr_plan_query(self.handle, Q_STATS, ctypes.cast(arr, ctypes.c_void_p),
                                            ctypes.sizeof(arr)), "sparsepr_plan_query")
        return [{f: getattr(s, f) for f, _ in HeadStats._fields_} for s in arr]
