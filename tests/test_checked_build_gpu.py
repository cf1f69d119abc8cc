"""The checked build on the GPU: libqlora_nf4_debug.so (QLORA_DEBUG) runs every
kernel family -- the quantizer, the dense dequantizer, the few-token, tiled and
CTA-pair forwards, the backward with its adapter and gradient kernels, dropout
and the merge -- with bounds and alignment checks before each TMA copy and
cluster exchange.  No check may fail, and every output must equal the ordinary
build's bit for bit (the checks change no arithmetic).  The checked library runs
in a child process (the binding picks it with QLORA_CHECKED_LIBRARY=1), so this
process keeps the ordinary one.
"""
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = """
import sys, json
import numpy as np, torch
sys.path.insert(0, {root!r})
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth

def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

out = {{}}
def keep(name, t):
    out[name] = t.detach().contiguous().view(torch.uint8).cpu().numpy() if t.dtype != torch.uint8 else t.cpu().numpy()

for (M, N, K, r, p) in [(1, 1024, 4096, 8, 0.0), (16, 640, 1024, 64, 0.0), (40, 512, 768, 16, 0.0),
                        (300, 512, 768, 64, 0.0), (300, 512, 768, 64, 0.3), (513, 1024, 1152, 24, 0.0)]:
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1500 + M)
    tag = "%d_%d_%d_%d_%g" % (M, N, K, r, p)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (dev(inp[k]) for k in ("X", "A", "B", "dY"))
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    if p > 0:
        Y = q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, inp["alpha"], p, 7, 3, U_save=U)
        g = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, inp["alpha"], p, 7, 3, dY, U_saved=U)
    else:
        Y = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, inp["alpha"], U_save=U)
        g = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, inp["alpha"], dY, U_saved=U)
    for name, t in (("codes", codes), ("q8", q8), ("s2", s2), ("Y", Y), ("U", U), ("dX", g[0]), ("dA", g[1]),
                    ("dB", g[2])):
        keep(tag + name, t)
    keep(tag + "deq", q.qlora_dequant(codes, q8, s2, N, K))
    keep(tag + "merge", q.qlora_merge_adapter(torch.from_numpy(inp["W"]).cuda(), A, B, inp["alpha"]))
torch.cuda.synchronize()
status = q.qlora_device_status()
record = q.qlora_debug_record() if {checked} else None
np.savez({path!r}, **out)
print(json.dumps({{"status": status, "record": record}}))
"""


def run(checked: bool, path: str) -> dict:
    import json
    env = dict(os.environ)
    env["QLORA_CHECKED_LIBRARY"] = "1" if checked else "0"
    code = CASES.format(root=ROOT, checked=checked, path=path)
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def test_checked_build_finds_nothing_and_matches_the_ordinary_build():
    from bit_nf4_quantized_quantize_b200 import build as qbuild
    qbuild.build()
    qbuild.build(debug=True)
    with tempfile.TemporaryDirectory() as d:
        a, b = os.path.join(d, "plain.npz"), os.path.join(d, "checked.npz")
        ra = run(False, a)
        rb = run(True, b)
        assert ra["status"] == 0 and rb["status"] == 0
        assert rb["record"] == {"failed": 0, "first_code": 0, "first_value": 0, "first_cta": 0}, rb["record"]
        pa, pb = np.load(a), np.load(b)
        assert sorted(pa.files) == sorted(pb.files) and len(pa.files) == 6 * 10
        for k in pa.files:
            assert np.array_equal(pa[k], pb[k]), k
