"""The guard-word build (libltxattn_debug.so, compiled with -DLTXATTN_DEBUG).

Its key-split calls put canary words around their fp32 partials and in every padded row
of the partial slabs, and check them on the device after the merge.  Each case runs in a
child process with LTXATTN_DEBUG=1 (which makes the binding load the debug library):
split calls of every kernel family must leave every guard intact and match the oracle;
with LTXATTN_DEBUG_CORRUPT_GUARD=1 the host overwrites one guard byte after the merge,
and ltxattn_check must report LTXATTN_ERR_WORKSPACE_GUARD, after which the context still
computes correct results.  No kernel faults or traps on either path.
"""
import os
import subprocess
import sys

import pytest

from joint_audio_video_flash_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from joint_audio_video_flash_b200 import ltxattn, synth
from oracle import oracle
assert ltxattn.LIB_PATH.endswith("libltxattn_debug.so")
torch.cuda.set_device(0)
ltxattn.create()
corrupt = sys.argv[2] == "corrupt"
# one query tile (two CTAs per SM), several query tiles (two per CTA, odd count: an empty
# second tile), head_dim 128; ragged query sides so that every slab has padded rows
cases = [(2, 4, 64, 126, 2048, 2000, 4), (1, 3, 64, 300, 3000, 2990, 5),
         (2, 2, 128, 200, 1500, 1400, 3), (1, 2, 128, 129, 4096, 4096, 16)]
for b, h, d, lq, lkv, valid, splits in cases:
    q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=lq + lkv, kv_valid=valid)
    out, used = ltxattn.forward(q.cuda(), k.cuda(), v.cuda(), kv_valid_len=valid,
                                num_splits=splits, return_splits=True)
    assert used > 1, used
    st = ltxattn.load().ltxattn_check(None)
    if corrupt:
        assert st == ltxattn.ERR_WORKSPACE_GUARD, ltxattn.status_string(st)
        break
    assert st == ltxattn.OK, ltxattn.status_string(st)
    ref = oracle.attention(q, k, v, d ** -0.5, kv_valid_len=valid)
    g = out.cpu().double().numpy()
    err = np.abs(g - ref).max()
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert err <= 2e-2 and rel <= 5e-3, (err, rel)
if corrupt:  # the word was cleared: an unsplit call afterwards is correct and clean
    q, k, v = synth.make_qkv(1, 300, 256, 2, 64, seed=3)
    out = ltxattn.forward(q.cuda(), k.cuda(), v.cuda())
    assert ltxattn.load().ltxattn_check(None) == ltxattn.OK
    ref = oracle.attention(q, k, v, 0.125)
    assert np.abs(out.cpu().double().numpy() - ref).max() <= 2e-2
print("debug-guards ok")
"""


@pytest.mark.parametrize("mode", ["clean", "corrupt"])
def test_guard_words(mode):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build(debug=True)
    env = dict(os.environ, LTXATTN_DEBUG="1")
    if mode == "corrupt":
        env["LTXATTN_DEBUG_CORRUPT_GUARD"] = "1"
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT, mode], capture_output=True,
                       text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "debug-guards ok" in r.stdout
