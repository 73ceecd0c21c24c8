"""Both ctypes bindings declare every function they load: a missing argtypes makes ctypes
pass 64-bit sizes as C ints, which silently corrupts the arguments."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_binding_declares_every_exported_function():
    import oracle
    src = open(os.path.join(ROOT, "oracle", "iqq_oracle.c"), encoding="utf-8").read()
    names = set(re.findall(r"^(?:int|float|double|void|int64_t|uint16_t)\s+(oracle_\w+)\(", src, re.M))
    assert names
    lib = oracle.lib()
    missing = [n for n in sorted(names) if getattr(lib, n).argtypes is None]
    assert not missing, missing


def test_library_binding_declares_every_header_function():
    import post_weight_quantization_rowwise_b200 as m
    src = open(os.path.join(ROOT, "include", "iqq.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(iqq_[a-z0-9_]+)\s*\(", src))
    missing = [n for n in sorted(names) if getattr(m._lib, n).argtypes is None]
    assert not missing, missing
