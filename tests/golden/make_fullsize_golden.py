"""Write the fp64 oracle's expected values for the two largest workloads.

At n = 32768 and n = 131072 one (b, h) instance of the fp64 oracle takes from seconds to
many minutes, too long to rerun inside every GPU test.  This script runs it once, on the
host, and stores what the GPU tests compare against:

  * the loss of every head (forward only for heads > 0) and their sum, the whole Loss;
  * the weight gradients dWQ, dWK, dWV of head 0 (B = 1, so one instance);
  * O, lse and the input gradients dA1, dA2, dA3 of instance (0, 0) at sampled query rows;
  * a SHA-256 digest of the seeded inputs, so a test can tell when the generator has drifted.

Only ``workloads`` (the seeded input generator) and ``oracle`` are used; nothing here
comes from the CUDA path.  Instances run in a process pool started with ``spawn``, one BLAS
thread per worker.

    python tests/golden/make_fullsize_golden.py [--jobs N] [workload ...]
    python tests/golden/make_fullsize_golden.py --approx-degree 1 b1_h8_n32768_d128_bf16_causal_bounded

With --approx-degree the approximate method's oracle values (the polynomial-kernel softmax of
that degree, see ``oracle.approx_instance_forward_backward``) are written instead.
"""
from __future__ import annotations

import argparse
import hashlib
import multiprocessing as mp
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))

NAMES = ["b1_h8_n32768_d128_bf16_causal_bounded", "b1_h8_n131072_d128_bf16_causal_base5e5"]
KEYS = ("A1", "A2", "A3", "E", "WQ", "WK", "WV", "pos")


def golden_path(name: str) -> str:
    return os.path.join(HERE, f"fullsize_{name}.npz")


def input_digest(inp) -> str:
    """SHA-256 over the raw bytes of the generated inputs, in a fixed key order."""
    h = hashlib.sha256()
    for k in KEYS:
        a = inp[k]
        h.update(k.encode())
        h.update(str(a.dtype).encode())
        h.update(repr(a.shape).encode())
        h.update(a.tobytes(order="C"))
    return h.hexdigest()


def sample_rows(n: int, count: int = 55, seed: int = 7):
    import numpy as np
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, n // 2, n - 129, n - 2, n - 1]
    rows = np.concatenate([fixed, rng.integers(0, n, count)])
    return np.unique(rows[(rows >= 0) & (rows < n)]).astype(np.int64)


def _instance(args):
    """One (0, h) instance: the full gradient when want_grad, else the loss only."""
    sys.path.insert(0, ROOT)
    import oracle
    h, sl, causal, base, want_grad, rows = args
    t0 = time.time()
    r = oracle.instance_forward_backward(sl["A1"], sl["A2"], sl["A3"], sl["E"], sl["WQ"],
                                         sl["WK"], sl["WV"], sl["pos"], causal, base,
                                         want_grad=want_grad)
    out = {"h": h, "loss": float(r["loss"]), "seconds": time.time() - t0}
    if want_grad:
        out.update({k: r[k] for k in ("dWQ", "dWK", "dWV")})
        out.update({k + "_rows": r[k][rows] for k in ("O", "lse", "dA1", "dA2", "dA3")})
    return out


def make(name: str, jobs: int) -> str:
    import numpy as np
    sys.path.insert(0, ROOT)
    from workloads import WORKLOADS, make_inputs
    w = WORKLOADS[name]
    assert w.B == 1, "the stored gradients are those of instance (0, h)"
    inp = make_inputs(w)
    digest = input_digest(inp)
    rows = sample_rows(w.n)
    tasks = []
    for h in range(w.H):
        sl = {k: np.ascontiguousarray(inp[k][0, h]) for k in ("A1", "A2", "A3", "E")}
        sl.update({k: np.ascontiguousarray(inp[k][h]) for k in ("WQ", "WK", "WV")})
        sl["pos"] = inp["pos"]
        tasks.append((h, sl, w.causal, w.rope_base, h == 0, rows))
    del inp
    t0 = time.time()
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(jobs, len(tasks))) as pool:
        res = sorted(pool.map(_instance, tasks, chunksize=1), key=lambda r: r["h"])
    g = res[0]
    loss_heads = np.array([r["loss"] for r in res], np.float64)
    path = golden_path(name)
    np.savez_compressed(
        path, workload=np.array(name), digest=np.array(digest), rows=rows,
        loss_heads=loss_heads, loss=np.array(float(np.sum(loss_heads))),
        dWQ=g["dWQ"], dWK=g["dWK"], dWV=g["dWV"],
        **{k + "_rows": g[k + "_rows"] for k in ("O", "lse", "dA1", "dA2", "dA3")})
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s "
          f"(per instance: {[round(r['seconds']) for r in res]} s)", flush=True)
    return path


def approx_path(name: str, degree: int) -> str:
    return os.path.join(HERE, f"fullsize_{name}_approx{degree}.npz")


def _approx_instance(args):
    sys.path.insert(0, ROOT)
    import oracle
    h, sl, causal, base, degree, rows = args
    t0 = time.time()
    r = oracle.approx_instance_forward_backward(sl["A1"], sl["A2"], sl["A3"], sl["E"], sl["WQ"],
                                                sl["WK"], sl["WV"], sl["pos"], causal, base,
                                                degree)
    out = {"h": h, "loss": float(r["loss"]), "seconds": time.time() - t0}
    if h == 0:
        out.update({k: r[k] for k in ("dWQ", "dWK", "dWV")})
        out["O_rows"] = r["O"][rows]
    return out


def make_approx(name: str, degree: int, jobs: int) -> str:
    """The approximate method's oracle values (polynomial degree ``degree``): the loss of every
    head, head 0's weight gradients and O at the sampled rows."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from workloads import WORKLOADS, make_inputs
    w = WORKLOADS[name]
    inp = make_inputs(w)
    digest = input_digest(inp)
    rows = sample_rows(w.n)
    tasks = []
    for h in range(w.H):
        sl = {k: np.ascontiguousarray(inp[k][0, h]) for k in ("A1", "A2", "A3", "E")}
        sl.update({k: np.ascontiguousarray(inp[k][h]) for k in ("WQ", "WK", "WV")})
        sl["pos"] = inp["pos"]
        tasks.append((h, sl, w.causal, w.rope_base, degree, rows))
    del inp
    t0 = time.time()
    with mp.get_context("spawn").Pool(min(jobs, len(tasks))) as pool:
        res = sorted(pool.map(_approx_instance, tasks, chunksize=1), key=lambda r: r["h"])
    g = res[0]
    loss_heads = np.array([r["loss"] for r in res], np.float64)
    path = approx_path(name, degree)
    np.savez_compressed(path, workload=np.array(name), digest=np.array(digest), rows=rows,
                        degree=np.array(degree), loss_heads=loss_heads,
                        loss=np.array(float(np.sum(loss_heads))), dWQ=g["dWQ"], dWK=g["dWK"],
                        dWV=g["dWV"], O_rows=g["O_rows"])
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s", flush=True)
    return path


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("names", nargs="*", default=NAMES)
    ap.add_argument("--jobs", type=int, default=len(os.sched_getaffinity(0)))
    ap.add_argument("--approx-degree", type=int, default=None,
                    help="write the approximate method's values (this degree) instead")
    a = ap.parse_args()
    # one BLAS thread per worker: the workers inherit these before importing numpy
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"
    for name in a.names:
        if a.approx_degree is None:
            make(name, a.jobs)
        else:
            make_approx(name, a.approx_degree, a.jobs)


if __name__ == "__main__":
    main()
