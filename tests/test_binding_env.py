"""Opt-in diagnostics of the Python binding (no GPU): NVTX ranges around every call
(MOE_NVTX=1) and a synchronising status check after every call (MOE_DEBUG_SYNC=1); both
leave the binding untouched when unset."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code, **env):
    e = dict(os.environ)
    e.pop("MOE_NVTX", None)
    e.pop("MOE_DEBUG_SYNC", None)
    e.update(env)
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=e, capture_output=True, text=True, timeout=120)


def test_nvtx_wrapping_is_opt_in():
    code = ("import sparse_moe_layer_joint_b200 as m; "
            "print(hasattr(m.moe_router_topk, '__wrapped__'), m.moe_permute_scratch_bytes(300, 256))")
    plain = _run(code)
    assert plain.returncode == 0, plain.stderr
    assert plain.stdout.split()[0] == "False"
    wrapped = _run(code, MOE_NVTX="1")
    assert wrapped.returncode == 0, wrapped.stderr
    assert wrapped.stdout.split() == ["True", plain.stdout.split()[1]]   # same results through the ranges


def test_debug_sync_flag():
    code = "import sparse_moe_layer_joint_b200 as m; print(m._DEBUG_SYNC)"
    assert _run(code).stdout.strip() == "False"
    assert _run(code, MOE_DEBUG_SYNC="1").stdout.strip() == "True"
