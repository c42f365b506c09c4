"""Host-side bookkeeping of bench.py: ncu traffic is reported only while the summary's
source hash matches the kernel source (CPU, no GPU)."""
import os

import bench


def _profile(root, name, digest, traffic="4.5e9"):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", name), "w") as f:
        f.write("# capture\n\n")
        f.write(f"source sha256[:16] of src/kernel.cu with its headers: {digest}\n\n")
        if traffic is not None:
            f.write(f"dram bytes per launch (read+write): {traffic}\n")


def test_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    root = str(tmp_path)
    os.makedirs(os.path.join(root, "src"))
    src = os.path.join(root, "src", "kernel.cu")
    with open(src, "w") as f:
        f.write("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", root)
    _profile(root, "k_cfg5.md", bench.source_digest(src))
    assert bench.profiled_traffic("k", "cfg5") == 4.5e9
    # the kernel changes after the capture: the counters no longer describe it
    with open(src, "w") as f:
        f.write("// kernel v2\n")
    assert bench.profiled_traffic("k", "cfg5") is None


def test_traffic_absent_without_summary_or_figure(tmp_path, monkeypatch):
    root = str(tmp_path)
    os.makedirs(os.path.join(root, "src"))
    src = os.path.join(root, "src", "kernel.cu")
    with open(src, "w") as f:
        f.write("// kernel\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("k", "cfg5") is None  # no summary at all
    _profile(root, "k_cfg5.md", bench.source_digest(src), traffic=None)
    assert bench.profiled_traffic("k", "cfg5") is None  # summary without the figure
    _profile(root, "k_cfg5.md", "0123456789abcdef")
    assert bench.profiled_traffic("k", "cfg5") is None  # hash of some other source


def test_committed_summaries_name_existing_sources():
    """Every committed ncu summary that bench.py reads names a source file of the repo."""
    import re
    pdir = os.path.join(bench.ROOT, "profiles")
    for name in os.listdir(pdir):
        text = open(os.path.join(pdir, name)).read()
        for m in re.finditer(r"source sha256\[:16\] of ([\w/.]+) with its headers:\s*([0-9a-f]{16})",
                             text):
            assert os.path.exists(os.path.join(bench.ROOT, m.group(1))), (name, m.group(1))


def test_traffic_goes_stale_when_an_included_header_changes(tmp_path, monkeypatch):
    """The digest covers the headers a kernel includes: a change to one of them (a barrier
    wait, a table layout) also retires the committed counters."""
    root = str(tmp_path)
    os.makedirs(os.path.join(root, "src"))
    os.makedirs(os.path.join(root, "include"))
    src = os.path.join(root, "src", "kernel.cu")
    with open(src, "w") as f:
        f.write('#include "local.cuh"\n#include "api.h"\n#include <cuda.h>\n// kernel\n')
    with open(os.path.join(root, "src", "local.cuh"), "w") as f:
        f.write("// wait limit 1 s\n")
    with open(os.path.join(root, "include", "api.h"), "w") as f:
        f.write("// layout v1\n")
    monkeypatch.setattr(bench, "ROOT", root)
    _profile(root, "k_cfg5.md", bench.source_digest(src))
    assert bench.profiled_traffic("k", "cfg5") == 4.5e9
    with open(os.path.join(root, "include", "api.h"), "w") as f:
        f.write("// layout v2\n")
    assert bench.profiled_traffic("k", "cfg5") is None
    _profile(root, "k_cfg5.md", bench.source_digest(src))
    assert bench.profiled_traffic("k", "cfg5") == 4.5e9
    with open(os.path.join(root, "src", "local.cuh"), "w") as f:
        f.write("// wait limit 2 s\n")
    assert bench.profiled_traffic("k", "cfg5") is None
