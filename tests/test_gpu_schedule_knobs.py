"""The GEMMs' schedule settings change timing, never results.

The library reads a few tuning settings from the environment once per process:
the lockstep windows (KDKL_SYNC_WINDOW, KDKL_SYNC_KWINDOW), the row-block group
size of split-major launches (KDKL_SPLIT_GROUP_MB), the column-group order of
the dHidden / dW tiles (KDKL_TILE_COL_GROUP), the die-aware numbering of the
CTA groups (KDKL_DIE_ORDER) and L2 eviction hints (KDKL_L2_HINTS).  Each only
reorders, delays or annotates the same work: every output element still has
exactly one writer and every partial result lands in the same slot, so loss,
lse, dHidden and dW (and the top-K producer's output) must be bit-identical
under any of them.  Each setting runs in a child process on a case that spans
several rounds of units, and the outputs must equal the default's bit for bit;
the default's lse and dHidden must match the oracle on sampled rows.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import synth
from oracle import kl as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# several rounds of 74 units in every GEMM kind, long enough reductions for the lockstep's
# checkpoints, row blocks of 1 MB (d = 2048) so that a 1 MB group holds one of them
SHAPE = dict(N=20000, d=2048, V=30011, K=32)
CHUNK = 3072

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import output_head_kl_b200 as K, synth
from tests import gpu_harness as H
s = dict(N=int(sys.argv[3]), d=int(sys.argv[4]), V=int(sys.argv[5]), K=int(sys.argv[6]))
x = synth.custom_inputs(s["N"], s["d"], s["V"], s["K"], seed=611, cache="zipf", logit_std=3.0, mask_frac=0.05,
                        w_std=0.05)
dx = H.to_device(x)
g = H.run_gpu(dx, chunk_tokens=int(sys.argv[7]))
ws = torch.empty(K.kdkl_teacher_topk_workspace_bytes(s["N"], s["d"], s["V"], s["K"]), dtype=torch.uint8,
                 device="cuda")
ti = torch.empty(s["N"], s["K"], dtype=torch.int32, device="cuda")
tv = torch.empty(s["N"], s["K"], dtype=torch.float32, device="cuda")
K.kdkl_teacher_topk(dx.hidden, dx.W, s["K"], ti, tv, ws)
torch.cuda.synchronize()
np.savez(sys.argv[2], loss=np.array([g.loss]), lse=g.lse, dH=g.dH, dW=g.dW, flags=np.array([g.flags]),
         ti=ti.cpu().numpy(), tv=tv.cpu().numpy())
'''

SETTINGS = {
    "default": {},
    "no_lockstep": {"KDKL_SYNC_WINDOW": "0", "KDKL_SYNC_KWINDOW": "0"},
    "tight_and_regrouped": {"KDKL_SYNC_WINDOW": "1", "KDKL_SYNC_KWINDOW": "8", "KDKL_SPLIT_GROUP_MB": "1",
                            "KDKL_TILE_COL_GROUP": "1", "KDKL_DIE_ORDER": "1", "KDKL_L2_HINTS": "3"},
}


def _run(tmp_path, name, env_extra):
    env = {k: v for k, v in os.environ.items() if not k.startswith("KDKL_")}
    env.update(env_extra)
    out = os.path.join(tmp_path, name + ".npz")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, out, *(str(SHAPE[k]) for k in ("N", "d", "V", "K")),
                        str(CHUNK)],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return dict(np.load(out))


def test_schedule_settings_do_not_change_results(tmp_path):
    res = {name: _run(str(tmp_path), name, env) for name, env in SETTINGS.items()}
    base = res["default"]
    for name, r in res.items():
        for key in ("loss", "lse", "dH", "dW", "flags", "ti", "tv"):
            np.testing.assert_array_equal(r[key], base[key], err_msg=f"{name}: {key}")
    # the shared result against the oracle on a seeded sample of rows (lse, dHidden)
    x = synth.custom_inputs(SHAPE["N"], SHAPE["d"], SHAPE["V"], SHAPE["K"], seed=611, cache="zipf", logit_std=3.0,
                            mask_frac=0.05, w_std=0.05)
    rows = synth.sample_rows(SHAPE["N"], 400, seed=612)
    ref = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, rows=rows, want_dW=False)
    H.assert_lse(base["lse"][rows], ref.lse)
    H.assert_grad(base["dH"][rows], ref.dH, "dHidden (sampled rows)")
    assert int(base["flags"][0]) == 0
