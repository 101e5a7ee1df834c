"""Batch-invariance harness: probe items run solo and embedded in larger batches, compared bit for bit.

Sources: "God Does Not Play Dice: Enforcing Batch Invariance in Agentic Kernel
Generation" (abstract) validates candidates dynamically, by checking that
outputs stay bitwise identical across batch contexts.  A comment on the
CoRun forum post ("You think you are measuring intelligence...") describes a
solo versus pad-batched A/B gate, logged with a pin tuple.  It also proposes
rerunning one fixed batch N times to bound run-to-run drift.

An *item* is what one request contributes to a batch: a row of activations, or
for decode attention a (query, keys, values) triple.  ``run_batch`` maps a list
of items to a list of per-item outputs (numpy arrays).  The harness never looks
inside items; it only arranges them and compares output bits.

Procedure (for each M in the sweep, ``trials`` times):
  * choose min(M, P) distinct random positions (seeded),
  * put probe p at the p-th chosen position and seeded filler items elsewhere,
  * run the batch and compare each probe's output bits with its solo (M = 1) output.
Each probe output whose bits differ in any position counts as one violation.
+0 and -0 differ.  Separately, ``rerun_check`` runs one fixed batch N times and
counts reruns whose bits differ from the first run.
"""
from __future__ import annotations

import datetime
import os
import platform
import subprocess
from dataclasses import dataclass, field
from typing import Callable, Sequence

import numpy as np

from . import inputs


def same_bits(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    return a.shape == b.shape and a.dtype == b.dtype and a.tobytes() == b.tobytes()


@dataclass
class BIReport:
    op: str
    violations: int = 0
    comparisons: int = 0
    rerun_violations: int = 0
    reruns: int = 0
    per_m: dict = field(default_factory=dict)
    first_failure: dict | None = None

    def as_dict(self):
        return {"op": self.op, "violations": self.violations, "comparisons": self.comparisons,
                "rerun_violations": self.rerun_violations, "reruns": self.reruns,
                "first_failure": self.first_failure}


def bi_check(op: str, run_batch: Callable[[list], list], probes: Sequence, filler: Callable[[int, int], object],
             m_list: Sequence[int], trials: int = 3, seed_positions: int = inputs.SEED_POSITIONS,
             report: BIReport | None = None) -> BIReport:
    """Count bitwise batch-invariance violations of `run_batch` over the M sweep.

    filler(trial, M) -> list of M deterministic filler items for that trial.
    """
    rep = report or BIReport(op)
    solo = [run_batch([p])[0] for p in probes]
    P = len(probes)
    for M in m_list:
        bad = 0
        for trial in range(trials):
            rng = np.random.default_rng([seed_positions, int(M), trial])
            pos = rng.choice(M, size=min(M, P), replace=False)
            batch = list(filler(trial, M))
            for p_idx, where in enumerate(pos):
                batch[int(where)] = probes[p_idx]
            out = run_batch(batch)
            for p_idx, where in enumerate(pos):
                rep.comparisons += 1
                if not same_bits(out[int(where)], solo[p_idx]):
                    bad += 1
                    if rep.first_failure is None:
                        diff = np.count_nonzero(np.ascontiguousarray(out[int(where)]).view(np.uint8) !=
                                                np.ascontiguousarray(solo[p_idx]).view(np.uint8))
                        rep.first_failure = {"M": int(M), "trial": trial, "position": int(where), "probe": p_idx,
                                             "differing_bytes": int(diff)}
        rep.per_m[int(M)] = bad
        rep.violations += bad
    return rep


def rerun_check(run_batch: Callable[[list], list], batch: list, n: int = 10, report: BIReport | None = None,
                op: str = "") -> BIReport:
    """Run one fixed batch n times; every rerun whose outputs differ in any bit from run 0 counts once."""
    rep = report or BIReport(op)
    ref = run_batch(batch)
    for _ in range(n - 1):
        out = run_batch(batch)
        rep.reruns += 1
        if not all(same_bits(a, b) for a, b in zip(out, ref)):
            rep.rerun_violations += 1
    return rep


def pin_tuple(extra: dict | None = None) -> dict:
    """What a result was produced with: GPU, driver, CUDA, torch, git commit, time."""
    d = {"host": platform.node(), "python": platform.python_version(),
         "utc": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds")}
    try:
        import torch
        d["torch"] = torch.__version__
        d["cuda_runtime"] = torch.version.cuda
        if torch.cuda.is_available():
            d["gpu"] = torch.cuda.get_device_name(0)
            cap = torch.cuda.get_device_capability(0)
            d["sm"] = f"{cap[0]}{cap[1]}"
    except Exception:  # pragma: no cover
        pass
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    try:
        d["git"] = subprocess.run(["git", "-C", root, "rev-parse", "--short", "HEAD"], capture_output=True,
                                  text=True, timeout=5).stdout.strip() or None
    except Exception:  # pragma: no cover
        d["git"] = None
    # the kernel sources themselves, for copies of the tree without version control
    import glob
    import hashlib
    hsh = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(root, "invariant_deterministic_rmsnorm_b200", "csrc", "*")) +
                    glob.glob(os.path.join(root, "include", "*.h"))):
        with open(f, "rb") as fh:
            hsh.update(fh.read())
    d["kernel_sources_sha256"] = hsh.hexdigest()[:16]
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=10).stdout.strip().splitlines()
        d["driver"] = out[0] if out else None
    except Exception:
        d["driver"] = None
    if extra:
        d.update(extra)
    return d


def bi_check_rows(op: str, run, probes, filler, m_list: Sequence[int], trials: int = 3,
                  seed_positions: int = inputs.SEED_POSITIONS, report: BIReport | None = None) -> BIReport:
    """Row-batch form of ``bi_check`` on torch tensors, batches assembled where the tensors live.

    run(batch [M, ...]) -> out [M, ...]; probes [P, ...]; filler(trial) -> tensor [>= max(m_list), ...].
    Outputs are compared as raw bits (viewed as integers of the same width).
    """
    import torch

    def bits(t):
        return t.contiguous().view({1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[t.element_size()])

    rep = report or BIReport(op)
    P = probes.shape[0]
    solo = [bits(run(probes[p:p + 1].clone())[0]).clone() for p in range(P)]
    for M in m_list:
        bad = 0
        for trial in range(trials):
            rng = np.random.default_rng([seed_positions, int(M), trial])
            pos = rng.choice(M, size=min(M, P), replace=False)
            batch = filler(trial)[:M].clone()
            for p_idx, where in enumerate(pos):
                batch[int(where)] = probes[p_idx]
            out = run(batch)
            for p_idx, where in enumerate(pos):
                rep.comparisons += 1
                if not torch.equal(bits(out[int(where)]), solo[p_idx]):
                    bad += 1
                    if rep.first_failure is None:
                        diff = int((bits(out[int(where)]) != solo[p_idx]).sum())
                        rep.first_failure = {"M": int(M), "trial": trial, "position": int(where), "probe": p_idx,
                                             "differing_elements": diff}
        rep.per_m[int(M)] = bad
        rep.violations += bad
    return rep


def rerun_check_rows(run, batch, n: int = 10, report: BIReport | None = None, op: str = "") -> BIReport:
    """Tensor form of ``rerun_check``: one fixed batch run n times, bitwise against the first run."""
    import torch
    rep = report or BIReport(op)
    ref = run(batch).clone()
    for _ in range(n - 1):
        out = run(batch)
        rep.reruns += 1
        if not torch.equal(out.contiguous().view(torch.uint8), ref.contiguous().view(torch.uint8)):
            rep.rerun_violations += 1
    return rep
