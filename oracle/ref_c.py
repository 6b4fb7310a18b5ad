"""Build and call the C oracle (oracle/h3ref.c) from Python.

TEST INFRASTRUCTURE, like the rest of oracle/: only the tests, the smoke
check and the benchmark's CPU baseline leg may use it. Two builds of the same
source: REAL = double ("f64") and REAL = float ("f32", the block in plain
fp32). gcc, no dependencies beyond libm.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "h3ref.c")
BUILD = os.path.join(HERE, "_build")


def lib_path(kind: str, build_dir: str = BUILD) -> str:
    return os.path.join(build_dir, f"libh3ref_{kind}.so")


def build(build_dir: str = BUILD, src: str = SRC, werror: bool = True) -> Dict[str, str]:
    """Compile both builds of `src` with gcc; returns {kind: path}."""
    cc = os.environ.get("CC") or shutil.which("gcc") or shutil.which("cc")
    if not cc:
        raise RuntimeError("no C compiler for the C oracle")
    os.makedirs(build_dir, exist_ok=True)
    out = {}
    for kind, defs in (("f64", []), ("f32", ["-DH3REF_REAL_FLOAT"])):
        path = lib_path(kind, build_dir)
        tmp = path + ".tmp"
        cmd = [cc, "-std=c99", "-O2", "-fPIC", "-shared", "-Wall", *(["-Werror"] if werror else []),
               *defs, src, "-o", tmp, "-lm"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"C oracle build failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, path)
        out[kind] = path
    return out


class Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("ffn", ctypes.c_int), ("sections", ctypes.c_int * 3), ("gelu_tanh", ctypes.c_int),
                ("theta", ctypes.c_double), ("eps", ctypes.c_double)]


class RefC:
    """One build of the C oracle. Arrays go in and come out as numpy, in the
    build's arithmetic type."""

    def __init__(self, path: str):
        self.lib = ctypes.CDLL(path)
        nbytes = self.lib.h3ref_real_bytes()
        self.real = {8: np.float64, 4: np.float32}[nbytes]
        P = ctypes.c_void_p
        self.lib.h3ref_token_positions.argtypes = [ctypes.c_int, P, ctypes.c_int, P]
        self.lib.h3ref_timestep_condition.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                                      ctypes.c_int, P, P, P, P, P]
        self.lib.h3ref_adaln.argtypes = [ctypes.c_int, P, P, P, P]
        self.lib.h3ref_block_forward.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int, P, P, P, P, P,
                                                 P, P, P]

    @staticmethod
    def _ptr(a: np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data_as(ctypes.c_void_p)

    def _r(self, a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=self.real)

    @staticmethod
    def _w(a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=np.float32)

    def token_positions(self, n_txt: int, grids: Sequence[Tuple[int, int, int]]) -> np.ndarray:
        g = np.ascontiguousarray(np.asarray(grids, dtype=np.int32).reshape(-1, 3))
        n = n_txt + int(sum(h * w for _, h, w in grids))
        pos = np.empty((n, 3), np.int32)
        self.lib.h3ref_token_positions(n_txt, self._ptr(g), len(g), self._ptr(pos))
        return pos

    def timestep_condition(self, t: float, tw: Dict[str, np.ndarray], dim: int = 256,
                           t_scale: float = 1000.0) -> np.ndarray:
        hidden = tw["b_t2"].shape[0]
        ws = [self._w(tw[k]) for k in ("w_t1", "b_t1", "w_t2", "b_t2")]
        c = np.empty(hidden, self.real)
        rc = self.lib.h3ref_timestep_condition(float(t), dim, float(t_scale), hidden,
                                               *[self._ptr(w) for w in ws], self._ptr(c))
        assert rc == 0
        return c

    def adaln(self, c, w_ada, b_ada) -> np.ndarray:
        c = self._r(c)
        hidden = c.shape[0]
        mod = np.empty(6 * hidden, self.real)
        w, b = self._w(w_ada), self._w(b_ada)
        assert self.lib.h3ref_adaln(hidden, self._ptr(c), self._ptr(w), self._ptr(b),
                                    self._ptr(mod)) == 0
        return mod.reshape(6, hidden)

    def block_forward(self, x, mod, w: Dict[str, np.ndarray], pos: np.ndarray, *, heads: int,
                      head_dim: int, sections: Sequence[int], gelu_tanh: bool = False,
                      theta: float = 1e4, eps: float = 1e-6) -> np.ndarray:
        x = self._r(x)
        n, hidden = x.shape
        ffn = w["w_ff1"].shape[0]
        cfg = Cfg(hidden, heads, head_dim, ffn, (ctypes.c_int * 3)(*sections), int(gelu_tanh),
                  theta, eps)
        m = self._r(np.asarray(mod).reshape(-1))
        ws = [self._w(w[k]) for k in ("w_qkv", "w_o", "w_ff1", "w_ff2")]
        p = np.ascontiguousarray(pos, dtype=np.int32)
        y = np.empty_like(x)
        rc = self.lib.h3ref_block_forward(ctypes.byref(cfg), n, self._ptr(x), self._ptr(m),
                                          *[self._ptr(a) for a in ws], self._ptr(p), self._ptr(y))
        assert rc == 0, "C oracle: bad sections or out of memory"
        return y


def load(kind: str = "f64", build_dir: Optional[str] = None) -> RefC:
    """The given build, compiled first if it is missing or older than the source."""
    d = build_dir or BUILD
    path = lib_path(kind, d)
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(SRC):
        build(d)
    return RefC(path)
