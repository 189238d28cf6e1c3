"""Static checks of the committed sources for constructs this library must never contain: TMA
loads with cluster multicast, the batched host/device copy calls, deliberate device traps or
asserts, and commands that change a GPU's settings.  CPU only (reads files)."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC_DIRS = [os.path.join(ROOT, "block_sparse_attention_pbsa_b200"), os.path.join(ROOT, "include")]
TOP_FILES = [os.path.join(ROOT, n) for n in ("bench.py", "__graft_entry__.py")]


def _files(exts):
    out = []
    for d in SRC_DIRS:
        for dp, _, names in os.walk(d):
            out += [os.path.join(dp, n) for n in names if n.endswith(exts)]
    return out + [p for p in TOP_FILES if p.endswith(exts)]


def _read(p):
    with open(p, encoding="utf-8", errors="replace") as fh:
        return fh.read()


def test_no_cluster_multicast_loads():
    for p in _files((".cu", ".cuh", ".h")):
        assert ".multicast::cluster" not in _read(p), p


def test_no_batched_copy_calls():
    # the names are assembled here so that this file does not contain them either
    names = [a + b for a in ("cudaMemcpy", "cudaMemcpy3D", "cuMemcpy", "cuMemcpy3D") for b in ("Batch" + "Async",)]
    for p in _files((".cu", ".cuh", ".h", ".py")):
        text = _read(p)
        for n in names:
            assert n not in text, (p, n)


def test_no_deliberate_device_traps():
    for p in _files((".cu", ".cuh")):
        text = _read(p)
        assert "__trap" not in text and not re.search(r"\btrap\s*;", text), p
        assert not re.search(r"^\s*assert\s*\(", text, flags=re.M), p


def test_gpu_settings_are_only_read():
    setters = ("-lgc", "-rgc", "-lmc", "-rmc", "-ac", "-rac", "-pm", "-pl", "-r", "--lock-gpu-clocks",
               "--reset-gpu-clocks", "--applications-clocks", "--persistence-mode", "--power-limit",
               "--gpu-reset", "-mig", "--compute-mode", "-c", "-e", "--ecc-config")
    seen = 0
    for p in _files((".py",)):
        for m in re.finditer(r"\[\s*\"nvidia-smi\"(.*?)\]", _read(p), flags=re.S):
            args = re.findall(r"\"([^\"]*)\"", m.group(1))
            assert any(a.startswith("--query") for a in args), (p, args)
            for a in args:
                assert a.split("=")[0] not in setters, (p, a)
            seen += 1
    assert seen >= 1   # the clock sampler of bench.py was inspected
