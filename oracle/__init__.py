"""fp64 CPU oracle of the hybrid-head sparse decode-attention step.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` leg (and its ``--impl reference`` arm) are the only
callers.  Nothing in ``hybrid_head_sparse_b200`` imports this package, and this
package imports nothing from it: the oracle shares no code with the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, fp64); this module compiles it
with gcc into ``liboracle.so`` next to it and wraps it with ctypes and numpy.
What it follows, from the page "LycheeDecode: Accelerating Long-Context LLM
Inference via Hybrid-Head Sparse Decoding" (paper-graph-ui summary):

* section 3.4 Eq. (1): a retrieval head attends over every cached row;
* section 3.4 Eq. (2): it selects the top-k rows as the next layer's set;
* section 3.4 Eq. (3): a sparse head attends over its inherited rows only
  and passes the set on unchanged;
* section 3.4 (propagation-chain initialisation) and Appendix B (Algorithm 1):
  every head of layer 0 is a retrieval head;
* section 3.4 "Hyperparameter summary": under GQA the queries of a KV group
  are averaged before token selection (``select_mode=1``);
* section 4.4.1 (Figure 6, Tables 5-6), section 4.1 / Appendix F and the
  kernel section: the selection rules other than a fixed k (ratio, the
  reasoning budget as the ratio 1/2, block top-k, top-p, threshold; see
  ``Selection`` and the readings at the top of oracle.c);
* section 4.2.2 (Cache Correction): the dense causal attention of the T most
  recent positions over the cache (``correction``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16 = 0
FP32 = 1
SELECT_PER_QHEAD = 0
SELECT_KVGROUP_MEAN = 1
RULE_TOPK = 0
RULE_RATIO = 1
RULE_BLOCK_TOPK = 2
RULE_TOPP = 3
RULE_THRESHOLD = 4


class OracleShape(ctypes.Structure):
    _fields_ = [
        ("L", ctypes.c_int),
        ("B", ctypes.c_int),
        ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("d", ctypes.c_int),
        ("n", ctypes.c_int64),
        ("dtype", ctypes.c_int),
        ("select_mode", ctypes.c_int),
        ("s_layer", ctypes.c_int64),
        ("s_batch", ctypes.c_int64),
        ("s_head", ctypes.c_int64),
        ("s_token", ctypes.c_int64),
    ]


class OracleSelection(ctypes.Structure):
    _fields_ = [
        ("rule", ctypes.c_int),
        ("block", ctypes.c_int),
        ("ratio_num", ctypes.c_int64),
        ("ratio_den", ctypes.c_int64),
        ("p", ctypes.c_double),
        ("tau", ctypes.c_double),
    ]


@dataclass
class Selection:
    """A selection rule (section 4.4.1, Figure 6, Tables 5-6; Appendix F):
    RULE_TOPK (fixed k), RULE_RATIO (ceil(num/den * n) rows), RULE_BLOCK_TOPK
    (whole blocks of `block` rows, scored by their summed probability),
    RULE_TOPP (smallest prefix reaching mass p), RULE_THRESHOLD (rows with
    probability >= tau).  Every rule keeps at most k rows."""
    rule: int = RULE_TOPK
    block: int = 64
    ratio: tuple = (1, 2)
    p: float = 0.9
    tau: float = 1e-3

    def c(self) -> OracleSelection:
        return OracleSelection(self.rule, self.block, int(self.ratio[0]), int(self.ratio[1]),
                               float(self.p), float(self.tau))


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, fp64, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        p = ctypes.c_void_p
        L.ora_topk.argtypes = [p, ctypes.c_int64, ctypes.c_int, p]
        L.ora_topk.restype = ctypes.c_int
        L.ora_layer.argtypes = [ctypes.POINTER(OracleShape), ctypes.c_int, p, p, p, p,
                                ctypes.c_int, ctypes.c_int, p, p, p, p, p]
        L.ora_layer.restype = ctypes.c_int
        L.ora_decode_step.argtypes = [ctypes.POINTER(OracleShape), p, p, p, p,
                                      ctypes.c_int, ctypes.c_int, p, p, p]
        L.ora_decode_step.restype = ctypes.c_int
        L.ora_select.argtypes = [p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(OracleSelection), p]
        L.ora_select.restype = ctypes.c_int
        L.ora_layer_sel.argtypes = [ctypes.POINTER(OracleShape), ctypes.POINTER(OracleSelection),
                                    ctypes.c_int, p, p, p, p, ctypes.c_int, ctypes.c_int, p, p,
                                    p, p, p]
        L.ora_layer_sel.restype = ctypes.c_int
        L.ora_decode_step_sel.argtypes = [ctypes.POINTER(OracleShape),
                                          ctypes.POINTER(OracleSelection), p, p, p, p,
                                          ctypes.c_int, ctypes.c_int, p, p, p]
        L.ora_decode_step_sel.restype = ctypes.c_int
        L.ora_correction.argtypes = [ctypes.POINTER(OracleShape), ctypes.c_int, p, p, p, p]
        L.ora_correction.restype = ctypes.c_int
        self.lib = L
        self.path = path

    def topk(self, x, k):
        return topk(x, k, self)

    def select(self, x, k, sel=None):
        return select(x, k, sel, self)

    def correction(self, *a, **kw):
        return correction(*a, ora=self, **kw)

    def layer(self, *a, **kw):
        return layer(*a, ora=self, **kw)

    def decode_step(self, *a, **kw):
        return decode_step(*a, ora=self, **kw)


_default: Oracle | None = None
_gomp = None


def _libgomp():
    """The OpenMP runtime the oracle library is linked with (one copy per
    process, so its thread setting applies to the oracle's parallel loops)."""
    global _gomp
    if _gomp is None:
        _gomp = ctypes.CDLL("libgomp.so.1")
        _gomp.omp_set_num_threads.argtypes = [ctypes.c_int]
        _gomp.omp_set_num_threads.restype = None
        _gomp.omp_get_max_threads.argtypes = []
        _gomp.omp_get_max_threads.restype = ctypes.c_int
    return _gomp


def max_threads() -> int:
    """Threads the oracle's next parallel loop uses."""
    default()
    return int(_libgomp().omp_get_max_threads())


def set_threads(n: int) -> None:
    """Threads for the oracle's parallel loops that this thread starts next
    (timing the oracle on one core against all cores)."""
    default()
    _libgomp().omp_set_num_threads(int(n))


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def compile_variant(source_text: str, out_path: str) -> Oracle:
    """Compile an edited copy of oracle.c (used by the tests that plant a
    mistake in the oracle to show that the pins catch it)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC", "-std=c11", "-o", out_path, src, "-lm"]
    subprocess.run(cmd, check=True)
    return Oracle(out_path)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


@dataclass
class Stack:
    """Host copies of one step's inputs, in the library's layouts.

    q    : [L][B][Hq][d]   uint16 (bf16 bit patterns) or float32
    k, v : [L][B][Hkv][n][d] same dtype (contiguous; strides derived)
    role : [L][Hq] uint8, 1 = retrieval
    """
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    role: np.ndarray
    select_mode: int = SELECT_PER_QHEAD

    def shape(self, n: int | None = None) -> OracleShape:
        # a cache row may be padded: the row stride is k.shape[-1], the head
        # dimension is q.shape[-1]
        L, B, Hkv, nmax, row = self.k.shape
        Hq, d = self.q.shape[2], self.q.shape[3]
        assert row >= d
        if self.k.dtype == np.uint16:
            dt = BF16
        elif self.k.dtype == np.float32:
            dt = FP32
        else:
            raise TypeError(f"unsupported cache dtype {self.k.dtype}")
        if not (self.k.flags.c_contiguous and self.v.flags.c_contiguous
                and self.q.flags.c_contiguous):
            raise ValueError("oracle inputs must be C-contiguous")
        return OracleShape(L, B, Hq, Hkv, d, nmax if n is None else n, dt,
                           self.select_mode, B * Hkv * nmax * row, Hkv * nmax * row,
                           nmax * row, row)

    @property
    def slots(self) -> int:
        return self.k.shape[2] if self.select_mode == SELECT_KVGROUP_MEAN else self.q.shape[2]


def topk(x: np.ndarray, k: int, ora: Oracle | None = None) -> np.ndarray:
    """argsTopK with ties to the lower index; ascending; -1 padded to k."""
    ora = ora or default()
    x = np.ascontiguousarray(x, dtype=np.float64)
    S = np.empty(k, dtype=np.int32)
    rc = ora.lib.ora_topk(_ptr(x), x.size, k, _ptr(S))
    if rc != 0:
        raise ValueError(f"ora_topk failed ({rc})")
    return S


def select(x: np.ndarray, k: int, sel: Selection | None = None,
           ora: Oracle | None = None) -> np.ndarray:
    """The set one selection rule picks from the keys x: ascending, -1 padded
    to k (sel None: top-k)."""
    ora = ora or default()
    x = np.ascontiguousarray(x, dtype=np.float64)
    S = np.empty(k, dtype=np.int32)
    cs = (sel or Selection()).c()
    rc = ora.lib.ora_select(_ptr(x), x.size, k, ctypes.byref(cs), _ptr(S))
    if rc != 0:
        raise ValueError(f"ora_select failed ({rc})")
    return S


def _sel_ref(sel: Selection | None):
    return None if sel is None else ctypes.byref(sel.c())


def layer(st: Stack, l: int, k: int, S_in: np.ndarray | None, all_retrieval: bool,
          n: int | None = None, ora: Oracle | None = None, sel: Selection | None = None):
    """One layer.  Returns (out [B][Hq][d] f64, S_out [B][Hs][k] i32,
    keys [B][Hs][n] f64 (valid for refreshed slots), refreshed [Hs] u8)."""
    sh = st.shape(n)
    B, Hq, d = sh.B, sh.Hq, sh.d
    Hs = st.slots
    out = np.zeros((B, Hq, d), dtype=np.float64)
    S_out = np.full((B, Hs, k), -1, dtype=np.int32)
    keys = np.zeros((B, Hs, sh.n), dtype=np.float64)
    fresh = np.zeros(Hs, dtype=np.uint8)
    if S_in is not None:
        S_in = np.ascontiguousarray(S_in, dtype=np.int32)
        assert S_in.shape == (B, Hs, k), S_in.shape
    role = np.ascontiguousarray(st.role, dtype=np.uint8)
    ora = ora or default()
    cs = (sel or Selection()).c()
    rc = ora.lib.ora_layer_sel(ctypes.byref(sh), ctypes.byref(cs), l, _ptr(st.q), _ptr(st.k),
                             _ptr(st.v), _ptr(role[l]), int(all_retrieval), k, _ptr(S_in),
                             _ptr(S_out), _ptr(out), _ptr(keys), _ptr(fresh))
    if rc != 0:
        raise ValueError(f"ora_layer failed ({rc})")
    return out, S_out, keys, fresh


def decode_step(st: Stack, k: int, S_in: np.ndarray | None = None, n: int | None = None,
                trace: bool = False, ora: Oracle | None = None, sel: Selection | None = None):
    """The whole L-layer step.  S_in given: S^(0) is S_in and role row 0 is
    obeyed; otherwise layer 0 is all retrieval.  Returns (out [L][B][Hq][d],
    S [B][Hs][k], trace [L][B][Hs][k] or None)."""
    sh = st.shape(n)
    L, B, Hq, d = sh.L, sh.B, sh.Hq, sh.d
    Hs = st.slots
    out = np.zeros((L, B, Hq, d), dtype=np.float64)
    S = np.full((B, Hs, k), -1, dtype=np.int32)
    if S_in is not None:
        S[...] = S_in
    tr = np.full((L, B, Hs, k), -1, dtype=np.int32) if trace else None
    role = np.ascontiguousarray(st.role, dtype=np.uint8)
    ora = ora or default()
    cs = (sel or Selection()).c()
    rc = ora.lib.ora_decode_step_sel(ctypes.byref(sh), ctypes.byref(cs), _ptr(st.q), _ptr(st.k),
                                   _ptr(st.v), _ptr(role), k, int(S_in is not None), _ptr(S),
                                   _ptr(out), _ptr(tr))
    if rc != 0:
        raise ValueError(f"ora_decode_step failed ({rc})")
    return out, S, tr


def correction(st: Stack, q: np.ndarray, ora: Oracle | None = None) -> np.ndarray:
    """Cache Correction's dense causal attention (section 4.2.2): q is
    [L][B][Hq][T][d] in the cache's dtype (bf16 as uint16 bit patterns); query
    t attends rows 0 .. n - T + t of st's cache.  Returns out [L][B][Hq][T][d] f64."""
    sh = st.shape()
    L, B, Hq, d = sh.L, sh.B, sh.Hq, sh.d
    q = np.ascontiguousarray(q)
    assert q.dtype == st.k.dtype and q.shape[:3] == (L, B, Hq) and q.shape[4] == d, q.shape
    T = q.shape[3]
    out = np.zeros((L, B, Hq, T, d), dtype=np.float64)
    ora = ora or default()
    rc = ora.lib.ora_correction(ctypes.byref(sh), T, _ptr(q), _ptr(st.k), _ptr(st.v), _ptr(out))
    if rc != 0:
        raise ValueError(f"ora_correction failed ({rc})")
    return out
