"""Test helper: build libfa_b200.so if needed, then import the binding."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_fa():
    spec = importlib.util.spec_from_file_location(
        "_fa_build", os.path.join(ROOT, "exact_io_aware_90_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import exact_io_aware_90_b200 as fa
    return fa
