"""The debug build (libstarattn_debug.so, -DSTAR_DEBUG): every global store the
kernels compute is checked against its buffer's size, a refused index is
recorded and skipped, nothing traps.

Each test runs in a fresh process that loads the debug build (STAR_ATTN_LIBRARY);
the parity cases run every kernel family on small shapes with canary-padded
outputs and must leave the record empty, the canaries intact and the results
within the oracle tolerances. The normal build's checks compile away."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_with_debug_build(body: str):
    from block_sparse_attention_phase_b200 import build
    path = build.build(debug=True)
    env = dict(os.environ, STAR_ATTN_LIBRARY=path, PYTHONPATH=ROOT)
    script = "import sys\nsys.path.insert(0, %r)\n" % ROOT + body
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return r.stdout


SELFTEST = r'''
import torch
import block_sparse_attention_phase_b200 as sa
assert sa.debug_build()
assert sa.debug_record() == (0, 0, 0, 0)
out = torch.zeros(17, dtype=torch.int32, device="cuda")
sa.selftest_bounds(out, 16)                 # index 16 against limit 16: refused
rec = sa.debug_record()
assert rec[0] == 1 and rec[1] > 0 and rec[2] == 16 and rec[3] == 16, rec
assert int(out[16]) == 0                    # the store was skipped
assert sa.device_status() == 5              # the bounds flag: STAR_ERR_CUDA, then cleared
assert sa.device_status() == 0 and sa.debug_record() == (0, 0, 0, 0)
print("ok")
'''

PARITY = r'''
import numpy as np, torch
import block_sparse_attention_phase_b200 as sa
import oracle, workloads
from tests.parity_util import check_rows, to_np
assert sa.debug_build()
CAN = 8  # canary elements on each side of every output (a multiple of 8: keeps 16-byte alignment)

def padded(shape, dtype):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * CAN, dtype=dtype, device="cuda")
    buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).fill_(0x5A5A if dtype == torch.bfloat16 else 0x5A5A5A5A)
    return buf, buf[CAN:CAN + n].view(shape)

def intact(buf, dtype):
    v = buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32)
    pat = 0x5A5A if dtype == torch.bfloat16 else 0x5A5A5A5A
    return bool((v[:CAN] == pat).all() and (v[-CAN:] == pat).all())

f = to_np
w = workloads.Workload("dbg", 2, 8, 2, 128, 1300, 512, 9, 2, 0, 3)
x = workloads.make_inputs(w, device="cuda")
B = w.block_size
# Phase 1
ob, o = padded((2, 1300, 8, 128), torch.bfloat16)
lb, l = padded((2, 8, 1300), torch.float32)
sa.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], B, o=o, lse=l)
ro, rl = oracle.phase1(f(x["q_ctx"]), f(x["k_ctx"]), f(x["v_ctx"]), B)
check_rows(f(o), ro, f(l), rl, "phase1")
assert intact(ob, torch.bfloat16) and intact(lb, torch.float32)
# a host's share with a separate anchor
oa, la = sa.phase1_anchored(x["q_ctx"][:, B:].contiguous(), x["k_ctx"][:, B:].contiguous(),
                            x["v_ctx"][:, B:].contiguous(), x["k_ctx"][:, :B].contiguous(),
                            x["v_ctx"][:, :B].contiguous(), B)
assert torch.equal(oa, o[:, B:]) and torch.equal(la, l[..., B:])
# query pass, then fused and two-kernel decode steps
cap = 16
kc = torch.full((2, cap, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
vc = kc.clone()
qb, oq = padded((2, 9, 8, 128), torch.bfloat16)
sa.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc, B, o=oq)
rq, rql = oracle.phase2_query(f(x["q_qry"]), f(x["k_qry"]), f(x["v_qry"]), f(x["k_ctx"]), f(x["v_ctx"]))
check_rows(f(oq), rq, None, None, "query")
assert intact(qb, torch.bfloat16)
kr = np.zeros((2, cap, 2, 128)); vr = np.zeros_like(kr)
kr[:, :9], vr[:, :9] = f(x["k_qry"]), f(x["v_qry"])
ws = sa.fused_decode_workspace(2, 8, 2, 128, 1300, B, "cuda")
for t, fn in enumerate((sa.phase2_decode_fused, sa.phase2_decode)):
    db, od = padded((2, 1, 8, 128), torch.bfloat16)
    kw = {"workspace": ws} if t == 0 else {}
    fn(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"], x["v_ctx"], kc, vc, 9 + t, B, o=od, **kw)
    rd, rdl, kr, vr = oracle.phase2_decode(f(x["q_dec"][t]), f(x["k_dec"][t]), f(x["v_dec"][t]),
                                           f(x["k_ctx"]), f(x["v_ctx"]), kr, vr, 9 + t)
    check_rows(f(od), rd, None, None, f"decode {t}")
    assert intact(db, torch.bfloat16)
# varlen Phase 1 and decode over two sequences
cu = [0, 700, 1300]
ov, lv = sa.phase1_varlen(x["q_ctx"][0], x["k_ctx"][0], x["v_ctx"][0], cu, B)
for i in range(2):
    ri, rli = oracle.phase1(f(x["q_ctx"][0][cu[i]:cu[i + 1]])[None], f(x["k_ctx"][0][cu[i]:cu[i + 1]])[None],
                            f(x["v_ctx"][0][cu[i]:cu[i + 1]])[None], B)
    check_rows(f(ov[cu[i]:cu[i + 1]]), ri[0], f(lv[:, cu[i]:cu[i + 1]]), rli[0], f"varlen {i}")
kv2 = torch.zeros((2, cap, 2, 128), dtype=torch.bfloat16, device="cuda")
vv2 = kv2.clone()
sa.phase2_decode_varlen(x["q_dec"][0], x["k_dec"][0], x["v_dec"][0], x["k_ctx"][0], x["v_ctx"][0], cu,
                        kv2, vv2, [0, 3], B)
torch.cuda.synchronize()
rec = sa.debug_record()
assert rec == (0, 0, 0, 0), rec
assert sa.device_status() == 0
print("ok")
'''


def test_debug_build_records_a_planted_violation_without_trapping():
    assert "ok" in _run_with_debug_build(SELFTEST)


def test_debug_build_every_kernel_family_stays_in_bounds():
    assert "ok" in _run_with_debug_build(PARITY)


def test_normal_build_compiles_the_checks_away():
    import os
    import torch
    import block_sparse_attention_phase_b200 as sa
    if os.environ.get("STAR_ATTN_LIBRARY"):
        pytest.skip("STAR_ATTN_LIBRARY names another build: this test is about the in-tree one")
    assert not sa.debug_build()
    out = torch.zeros(5, dtype=torch.int32, device="cuda")
    sa.selftest_bounds(out, 4)  # no check: the (in-bounds) store of element 4 happens
    assert int(out[4]) == 1
    assert sa.debug_record() == (0, 0, 0, 0) and sa.device_status() == 0
