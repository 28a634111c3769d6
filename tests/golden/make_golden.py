"""Write oracle outputs for sampled subsets of the large workloads (CPU only).

Calls nothing but the CPU oracle and the seeded generators.  Each file holds, for the
listed sequences of the workload and its first `steps` tokens (float32 oracle):
  seqs      sequence indices within the batch
  logp_tok  [n, steps]  log p(x_{t+1} | x_{<=t}) at the workload's temperature (0 at t = T)
  lse       [n, steps]  log-sum-exp of the head at that temperature
  s_idx     steps at which s_t is stored (1-based)
  s         [n, len(s_idx), d]  s_t at those steps
  score     [n]  replay score over the response part of the first `steps` tokens
  prompt_len, steps, tau

    python tests/golden/make_golden.py 300m-12+12-b512 --seqs 0 1 2 3 --steps 256
"""
from __future__ import annotations

import argparse
import sys
import time
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
sys.path.insert(0, str(HERE.parent.parent))

from oracle import RLTOracle  # noqa: E402
from workloads import WORKLOADS, make_tokens, make_weights  # noqa: E402


def golden_path(workload: str, tag: str) -> Path:
    return HERE / f"oracle_{workload}_{tag}.npz"


def make(workload: str, seqs: list[int], steps: int, tag: str, s_every: int = 16) -> Path:
    wl = WORKLOADS[workload]
    m = wl.model
    t0 = time.time()
    w = make_weights(m, wl.weight_seed)
    ora = RLTOracle(m, w, np.float32)
    del w
    tok = make_tokens(wl, seqs)[:, :steps]
    e, M = ora.encode(tok)
    st = ora.init_state(len(seqs))
    n = len(seqs)
    logp_tok = np.zeros((n, steps), np.float32)
    lse = np.zeros((n, steps), np.float32)
    s_idx = sorted(set(list(range(s_every, steps + 1, s_every)) + [1, steps]))
    s_keep = []
    for t in range(1, steps + 1):
        st, logp = ora.step(st, e[:, t - 1], M, wl.tau)
        zt = ora._lin(ora.rnd(st.s), ora.w["unembed"]) / wl.tau
        mx = zt.max(-1, keepdims=True)
        lse[:, t - 1] = (mx + np.log(np.exp(zt - mx).sum(-1, keepdims=True)))[:, 0]
        if t < wl.T and t < tok.shape[1]:
            logp_tok[:, t - 1] = logp[np.arange(n), tok[:, t]]
        if t in s_idx:
            s_keep.append(st.s.copy())
        if t % 64 == 0:
            print(f"{workload}: step {t}/{steps} ({time.time() - t0:.0f}s)", flush=True)
    P = wl.prompt_len
    ts = np.arange(1, steps + 1)
    scored = (ts >= P) & (ts < min(steps, wl.T))
    score = (logp_tok * scored[None, :]).sum(-1)
    out = golden_path(workload, tag)
    np.savez_compressed(out, seqs=np.array(seqs), logp_tok=logp_tok, lse=lse, s_idx=np.array(s_idx),
                        s=np.stack(s_keep, 1).astype(np.float32), score=score.astype(np.float32),
                        prompt_len=P, steps=steps, tau=wl.tau)
    print(f"wrote {out} in {time.time() - t0:.0f}s", flush=True)
    return out


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=sorted(WORKLOADS))
    ap.add_argument("--seqs", type=int, nargs="+", default=[0, 1, 2, 3])
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--tag", default=None)
    ap.add_argument("--s-every", type=int, default=16)
    a = ap.parse_args()
    tag = a.tag or f"{len(a.seqs)}x{a.steps}"
    make(a.workload, a.seqs, a.steps, tag, a.s_every)
    return 0


if __name__ == "__main__":
    sys.exit(main())
