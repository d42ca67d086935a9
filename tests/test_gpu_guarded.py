"""The guarded debug build (libratp_guarded.so: every global access a kernel
addresses itself is range-checked; an out-of-range access is skipped and
reported as RATP_ERR_BOUNDS) stands in for a memory checker.  The small GPU
parity tests run again against it in a child process: any refused access
raises through ratp.last_error() in those tests and fails them."""
import os
import re
import subprocess
import sys

import pytest

from recurrence_augmented_dilated_chunked_b200 import build as B

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SMALL_TESTS = ["tests/test_gpu_scan.py", "tests/test_gpu_chunk_local.py", "tests/test_gpu_window.py",
               "tests/test_gpu_attn.py", "tests/test_gpu_per_sample.py", "tests/test_gpu_decode.py",
               "tests/test_gpu_layers.py", "tests/test_gpu_fused.py"]


def _env(**extra):
    env = dict(os.environ, **extra)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    return env


def _child(args, timeout):
    env = _env(RATP_LIBRARY=B.build_library(guarded=True))
    return subprocess.run([sys.executable] + args, cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_guard_refuses_an_out_of_range_access():
    code = ("import ctypes, recurrence_augmented_dilated_chunked_b200 as r\n"
            "from recurrence_augmented_dilated_chunked_b200._binding import RatpError\n"
            "import torch; torch.cuda.init()\n"
            "lib = r.load_library()\n"
            "assert r.guard_line() == (True, 0)\n"
            "assert lib.ratp_debug_guard_probe(None) == 0\n"
            "try:\n    r.last_error(); raise SystemExit('no error recorded')\n"
            "except RatpError as e:\n    assert e.code == 8, e.code\n"
            "guarded, line = r.guard_line()\n"
            "assert guarded and line > 0, line\n"
            "print('guard ok', line)\n")
    res = _child(["-c", code], 300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "guard ok" in res.stdout


def test_small_parity_suite_under_the_guarded_build():
    res = _child(["-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                  "-k", "not full_size and not beyond_2_pow_31 and not largest"] + SMALL_TESTS, 1800)
    tail = "\n".join((res.stdout + res.stderr).splitlines()[-30:])
    assert res.returncode == 0, tail
    m = re.search(r"(\d+) passed", res.stdout)
    assert m and int(m.group(1)) >= 200, tail


_SAME_BITS = r"""
import sys, torch
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import prefill_inputs
dev = "cuda"
B, T, H, Dh, n = 2, 300, 2, 128, 3
q, xk, xv, g = (x.to(dev) for x in prefill_inputs(B, T + n, H, Dh, "bf16", seed=5))
pre = [x[:, :T].contiguous() for x in (xk, xv, g)]
st = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=dev)
hk, hv = ratp.scan_prefill_kv(*pre, final_state=st)
o = ratp.dilated_attn_prefill(q[:, :T].contiguous(), hk, hv, 4, 16, head_mask=[1, 0])
wk, wv = ratp.scan_prefill_kv_window(*pre, 32)
cache = ratp.KVCache(B, H, Dh, T + n, 4, 16, head_mask=[1, 0])
cache.pack(hk, hv)
outs = [cache.decode_step(*[x[:, T + i].contiguous() for x in (q, xk, xv, g)], st) for i in range(n)]
ratp.last_error()
torch.save({"hk": hk.cpu(), "o": o.cpu(), "wk": wk.cpu(), "st": st.cpu(),
            "dec": torch.stack(outs).cpu()}, sys.argv[1])
"""


def test_guarded_build_computes_the_same_bits(tmp_path):
    """The range checks change no arithmetic: scan, attention, look-back scan
    and decode give bit-identical results in both builds."""
    import torch
    script = tmp_path / "same_bits.py"
    script.write_text(_SAME_BITS)
    res = _child([str(script), str(tmp_path / "guarded.pt")], 300)
    assert res.returncode == 0, res.stdout + res.stderr
    env = _env()
    env.pop("RATP_LIBRARY", None)
    res2 = subprocess.run([sys.executable, str(script), str(tmp_path / "normal.pt")], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)
    assert res2.returncode == 0, res2.stdout + res2.stderr
    a, b = torch.load(tmp_path / "guarded.pt"), torch.load(tmp_path / "normal.pt")
    for k in a:
        assert torch.equal(a[k].view(torch.uint8) if a[k].dtype == torch.bfloat16 else a[k],
                           b[k].view(torch.uint8) if b[k].dtype == torch.bfloat16 else b[k]), k
