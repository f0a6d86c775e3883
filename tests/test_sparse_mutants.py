"""The sparse oracle's pins must catch plausible mistakes.

Each case plants one slip in a copy of oracle/sparse.py (in a temporary
directory) and runs tests/test_sparse_oracle.py against that copy in a child
process: the pins have to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sparse.py")

MUTANTS = {
    "codes truncated, not rounded": ("k8 = np.clip(np.rint(kp / sk[..., None, None])",
                                     "k8 = np.clip(np.floor(kp / sk[..., None, None])"),
    "block scale over 128": ("sk = np.where(amax > 0, amax / np.float32(127.0)",
                             "sk = np.where(amax > 0, amax / np.float32(128.0)"),
    "padding rows not zeroed": ("kf[~np.broadcast_to(valid[:, None, :, None], kf.shape)] = 0.0",
                                "pass"),
    "one query scale per tensor": ("    amax = np.abs(qf).max(axis=-1)\n",
                                   "    amax = np.broadcast_to(np.abs(qf).max(), qf.shape[:-1])\n"),
    "strict threshold": ("(bmax[s0:s1] >= thr[None, :])", "(bmax[s0:s1] > thr[None, :])"),
    "one threshold for the whole history": (
        "M = bmax[s0:s1].max(axis=0)", "M = bmax.max(axis=0)"),
    "first head of the group only": ("(bmax[s0:s1] >= thr[None, :]).any(axis=1)",
                                     "(bmax[s0:s1] >= thr[None, :])[:, 0]"),
    "delta added, not subtracted": ("thr = (M - delta32)", "thr = (M + delta32)"),
    "equal chunks of ceil(T / S) blocks": (
        "return [(s * T // S, (s + 1) * T // S) for s in range(S)]",
        "return [(s * -(-T // S), min(T, (s + 1) * -(-T // S))) for s in range(S)]"),
    "kept blocks ignored in attention": ("tok = tok[kept[b, h, tok // BLOCK]]", "pass"),
    # the fp64 form of the selection (select_blocks_exact / block_maxima_exact)
    "exact: query scale dropped": (
        "factor = sc * sq[b, h * G:(h + 1) * G].astype(np.float64)",
        "factor = sc * np.ones(G)"),
    "exact: first block's scale for every block": (
        "logit = factor[None, :] * sk[b, h, blk].astype(np.float64)[:, None] * dots",
        "logit = factor[None, :] * float(sk[b, h, 0]) * dots"),
    "exact: whole history as one split": (
        "        for s0, s1 in split_blocks(L, num_splits):\n            if s0 >= nb:\n"
        "                break\n            s1 = min(nb, s1)\n            part = bm[s0:s1]",
        "        for s0, s1 in [(0, nb)]:\n            if s0 >= nb:\n"
        "                break\n            s1 = min(nb, s1)\n            part = bm[s0:s1]"),
    "exact: certainty against the split maximum": (
        "other = np.where(np.arange(n_blk)[:, None] == top[None, :], second[None, :],",
        "other = np.where(np.arange(n_blk)[:, None] == top[None, :], m1[None, :],"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not found once"
    path = tmp_path / "sparse_mutant.py"
    path.write_text(src.replace(old, new))
    env = dict(os.environ, FD_SPARSE_ORACLE=str(path))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_sparse_oracle.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch mutant '{name}':\n{r.stdout[-2000:]}"
