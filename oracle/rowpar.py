"""All-cores timing of the oracle: the same single-threaded C oracle, run in
one process per host core on disjoint row blocks of one weight matrix.

Test infrastructure, like the rest of oracle/: only tests/, the smoke check
and bench.py's CPU-baseline leg use it.  Nothing here changes the oracle's
arithmetic; each worker calls oracle.matmul_i32 and oracle.rescale on its rows.

Protocol (one worker per process, started with `python -m oracle.rowpar`):
  argv: shm_codes M K shm_q N row_begin row_end alpha shm_amax reps
  the worker attaches the shared-memory blocks, prints "ready", waits for one
  line on stdin, computes acc = codes[rb:re] x q^T and y = rescale(acc) `reps`
  times, prints "t0 t1" (time.monotonic, comparable across processes) and
  exits.
"""
import os
import subprocess
import sys
import time
from multiprocessing import shared_memory

import numpy as np


def _attach(name):
    """Attach to the parent's block without adopting it: on this Python an
    attaching process registers the block with its resource tracker, which
    would unlink it when the worker exits."""
    from multiprocessing import resource_tracker
    shm = shared_memory.SharedMemory(name=name)
    try:
        resource_tracker.unregister(shm._name, "shared_memory")
    except Exception:  # noqa: BLE001
        pass
    return shm


def _worker(argv):
    import oracle
    (name_c, M, K, name_q, N, rb, re_, alpha, name_a, reps) = argv
    M, K, N, rb, re_ = int(M), int(K), int(N), int(rb), int(re_)
    shm_c = _attach(name_c)
    shm_q = _attach(name_q)
    shm_a = _attach(name_a)
    try:
        codes = np.ndarray((M, K), np.int8, buffer=shm_c.buf)
        q = np.ndarray((N, K), np.int8, buffer=shm_q.buf)
        amax = np.ndarray((N,), np.float32, buffer=shm_a.buf)
        block = np.ascontiguousarray(codes[rb:re_])
        oracle.lib()
        print("ready", flush=True)
        sys.stdin.readline()
        t0 = time.monotonic()
        for _ in range(int(reps)):
            acc = oracle.matmul_i32(block, q)
            oracle.rescale(acc, np.float32(alpha), amax)
        t1 = time.monotonic()
        print("%.9f %.9f" % (t0, t1), flush=True)
        del codes, q, amax, block
    finally:
        shm_c.close()
        shm_q.close()
        shm_a.close()


def time_all_cores(codes, q, amax, alpha, reps=1, workers=None):
    """Time acc = codes x q^T (+ rescale), `reps` times over, on `workers`
    processes (default: every online core), each on a contiguous block of
    rows.  Returns (seconds from the first start to the last finish, workers
    used)."""
    workers = workers or os.cpu_count() or 1
    M, K = codes.shape
    N = q.shape[0]
    workers = max(1, min(workers, M))
    blocks = []
    shms = []
    try:
        for arr in (codes, q, amax.astype(np.float32)):
            shm = shared_memory.SharedMemory(create=True, size=max(1, arr.nbytes))
            np.ndarray(arr.shape, arr.dtype, buffer=shm.buf)[...] = arr
            shms.append(shm)
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        procs = []
        for w in range(workers):
            rb, re_ = M * w // workers, M * (w + 1) // workers
            blocks.append((rb, re_))
            procs.append(subprocess.Popen(
                [sys.executable, "-m", "oracle.rowpar", shms[0].name, str(M), str(K),
                 shms[1].name, str(N), str(rb), str(re_), repr(float(alpha)), shms[2].name,
                 str(int(reps))],
                cwd=root, stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True))
        for p in procs:
            if p.stdout.readline().strip() != "ready":
                raise RuntimeError("oracle worker failed to start")
        for p in procs:
            p.stdin.write("go\n")
            p.stdin.flush()
        starts, ends = [], []
        for p in procs:
            t0, t1 = (float(v) for v in p.stdout.readline().split())
            starts.append(t0)
            ends.append(t1)
            p.wait()
        return max(ends) - min(starts), workers
    finally:
        for shm in shms:
            shm.close()
            shm.unlink()


if __name__ == "__main__":
    _worker(sys.argv[1:])
