"""The bounds-checked build (libmxmoe_debug.so, -DMX_DEBUG_BOUNDS) on the GPU.

In that build every kernel index the checks cover (routing writes, the
dispatch-gradient rows, the requantisation's loads and stores, the grouped
GEMMs' scale-atom loads and outer scales, the NVFP4-backward loads and stores)
is compared with the extent the call's arguments give its buffer; an access
out of range is skipped and counted.  A child process with MX_DEBUG=1 runs the
tiny layer's forward and backward in both backward formats plus ragged
requantisations, routing with empty experts, and grouped GEMMs with 200 experts
of one or three row tiles (enough leftover tiles for the row-mode tail kernel);
it must count no violation and produce the same bytes as the normal build.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
from fp8_moe_numerics_b200 import api, workloads
from fp8_moe_numerics_b200 import _lib
from fp8_moe_numerics_b200.layer import ExpertLayer

def run():
    out = {}
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    for fmt in ("mxfp8", "nvfp4"):
        L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(), inp["w2"].cuda(),
                        inp["dout"].cuda(), gated=False, seed=3, wgrad_dtype=torch.float32, backward=fmt)
        L.step()
        api.sync_status()
        for n in ("out", "dx", "dw1", "dw2"):
            out[fmt + "_" + n] = getattr(L, n).float().cpu().numpy()
    ids = workloads.routing(700, 8, 64, "zipf", 1.2, 5, seed=4).cuda()
    seg, src, pos = api.moe_route(ids, 64)
    out["seg"], out["src"], out["pos"] = seg.cpu().numpy(), src.cpu().numpy(), pos.cpu().numpy()
    for R in (8, 16, 32):
        x = workloads.activations(384, 192, "t4_rowscale", 5 + R, "cuda")
        q = api.nvfp4_quantize(x, 1, api.MX_SF_MMA)
        oc, oe = api.mxfp8_requant_transpose_sr(*q, 384, 192, 1, api.MX_SF_MMA, None, 1, 2, R, api.MX_SF_ROWMAJOR)
        out[f"rq{R}"] = oc.cpu().numpy()
        out[f"rq{R}_e"] = oe.cpu().numpy()
    # grouped GEMMs whose leftover row tiles go to the tail kernel: 200 experts of 1 or 3 row tiles,
    # 4 column tiles of 256 (800 leftover tiles); valid random codes and scales
    counts = [60 + 200 * (i % 2) for i in range(200)]
    seg2 = torch.tensor(np.concatenate([[0], np.cumsum([(c + 127) // 128 * 128 for c in counts])]),
                        dtype=torch.int64).cuda()
    E2, N2, K2, valid = 200, 1024, 256, int(seg2[-1])
    M2 = valid + 128
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    u8 = lambda n, lo=0, hi=256: torch.randint(lo, hi, (n,), dtype=torch.uint8, device="cuda", generator=g)
    a = (u8(M2 * K2 // 2).view(M2, K2 // 2), u8(api.sf_bytes(M2, K2, 16, api.MX_SF_MMA), 0x30, 0x48),
         torch.full((M2,), 1e-2, device="cuda"))
    b = (u8(E2 * N2 * K2 // 2).view(E2 * N2, K2 // 2), u8(api.sf_bytes(E2 * N2, K2, 16, api.MX_SF_MMA), 0x30, 0x48),
         torch.full((E2,), 1e-2, device="cuda"))
    out["gemm_nvfp4_tail"] = api.grouped_gemm_nvfp4(a, b, seg2, E2, N2, K2).float().cpu().numpy()[:valid]
    ac = u8(M2 * K2).view(M2, K2) & 0x77
    bc = u8(N2 * E2 * K2).view(N2, E2 * K2) & 0x77
    ae = u8(api.sf_bytes(M2, K2, 32, api.MX_SF_MMA), 120, 134)
    be = u8(api.sf_bytes(N2, E2 * K2, 32, api.MX_SF_MMA), 120, 134)
    out["gemm_mxfp8_tail"] = api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, ac, ae, bc, be, seg2, E2, M2, N2,
                                                     K2).float().cpu().numpy()[:valid]
    api.sync_status()
    torch.cuda.synchronize()
    return out

res = run()
np.savez(OUT, **res)
print(json.dumps({"debug_build": _lib.lib().mx_debug_bounds_build(),
                  "violations": int(_lib.lib().mx_debug_bounds_violations(1))}))
"""


@pytest.fixture(scope="module")
def debug_lib():
    from fp8_moe_numerics_b200 import build
    return build.build(debug_bounds=True)


def test_bounds_checked_build_counts_nothing_and_matches(cuda, debug_lib, tmp_path):
    outs = {}
    reports = {}
    for mode in ("0", "1"):
        path = str(tmp_path / f"out{mode}.npz")
        code = CHILD.replace("ROOT", repr(ROOT)).replace("OUT", repr(path))
        env = dict(os.environ, MX_DEBUG=mode)
        p = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stderr[-3000:]
        reports[mode] = json.loads(p.stdout.strip().splitlines()[-1])
        outs[mode] = dict(np.load(path))
    assert reports["0"] == {"debug_build": 0, "violations": 0}
    assert reports["1"] == {"debug_build": 1, "violations": 0}
    assert outs["0"].keys() == outs["1"].keys()
    for k in outs["0"]:
        assert np.array_equal(outs["0"][k], outs["1"][k]), k
