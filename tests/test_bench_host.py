"""Host logic of bench.py (CPU): the committed per-launch DRAM traffic is reported only while
the forward kernels' sources are the ones it was captured from."""
import importlib.util
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _copy_tree(tmp_path, b):
    """The kernel sources in a scratch tree, with a traffic file written for them (the committed
    figures belong to the capture's sources, which later edits may have left behind)."""
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "fine_grained_mixture_moe_b200", "csrc"),
                    root / "fine_grained_mixture_moe_b200" / "csrc")
    (root / "profiles").mkdir()
    b.ROOT = str(root)
    with open(root / "profiles" / "traffic_quartz.txt", "w") as fh:
        fh.write("# test figures\n")
        fh.write(f"sources_sha256 {b.kernel_sources_sha256()}\n")
        fh.write("gemm_gateup 148840960\n")
    return root


def test_traffic_follows_the_forward_sources(tmp_path):
    b = _bench()
    _copy_tree(tmp_path, b)
    got = b.captured_traffic("quartz", "gemm_gateup")
    assert got == 148840960
    assert b.captured_traffic("quartz", "no_such_kernel") is None
    assert b.captured_traffic("no_such_workload", "gemm_gateup") is None
    csrc = os.path.join(b.ROOT, "fine_grained_mixture_moe_b200", "csrc")
    # the backward kernels are not part of the step: editing them keeps the figures
    with open(os.path.join(csrc, "backward.cuh"), "a") as fh:
        fh.write("\n// edited\n")
    assert b.captured_traffic("quartz", "gemm_gateup") == got
    # a forward kernel's source changed: the figures no longer apply
    with open(os.path.join(csrc, "gemm_tc2.cuh"), "a") as fh:
        fh.write("\n// edited\n")
    assert b.captured_traffic("quartz", "gemm_gateup") is None
