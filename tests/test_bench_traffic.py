"""The DRAM traffic that bench.py reports comes from an ncu summary under
profiles/, and only while the kernel's sources are those the counters were
taken from.  The sources are compared by a sha256 that ignores comments and
whitespace and nothing else."""

import os
import shutil

import bench

KERNEL = "decode_kernel"
WORKLOAD = "some-workload"


def _tree(tmp_path):
    """A copy of the kernel's sources and an empty profiles/ under tmp_path."""
    src = os.path.join(tmp_path, "lora_shared_kv_b200", "csrc")
    os.makedirs(src)
    for name in bench.KERNEL_SOURCES[KERNEL]:
        shutil.copy(os.path.join(bench.ROOT, "lora_shared_kv_b200", "csrc", name), src)
    os.makedirs(os.path.join(tmp_path, "profiles"))
    return src


def _edit(path, old, new):
    with open(path) as f:
        s = f.read()
    assert old in s
    with open(path, "w") as f:
        f.write(s.replace(old, new, 1))


def _summary(tmp_path, sha, nbytes):
    with open(os.path.join(tmp_path, "profiles", f"{KERNEL}__{WORKLOAD}.md"), "w") as f:
        f.write(f"# {KERNEL}\n\n- sources_sha256: `{sha}`\n- dram_bytes_per_launch: `{nbytes}`\n")


def test_hash_ignores_comments_and_layout_only(tmp_path, monkeypatch):
    src = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_sha256(KERNEL)
    decode = os.path.join(src, "decode.cu")
    _edit(decode, "namespace lrkv {", "// a new comment\n/* and a block\n   comment */\nnamespace   lrkv\n{")
    assert bench.kernel_sources_sha256(KERNEL) == h0
    _edit(decode, "constexpr int SEG_CHUNK = 8;", "constexpr int SEG_CHUNK = 4;")
    assert bench.kernel_sources_sha256(KERNEL) != h0


def test_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    src = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic(KERNEL, WORKLOAD) is None            # no summary
    _summary(tmp_path, bench.kernel_sources_sha256(KERNEL), 123456789)
    assert bench.profiled_traffic(KERNEL, WORKLOAD) == 123456789
    _edit(os.path.join(src, "lrkv_internal.h"), "constexpr uint32_t kSpinCap = 1u << 24;",
          "constexpr uint32_t kSpinCap = 1u << 23;")
    assert bench.profiled_traffic(KERNEL, WORKLOAD) is None            # the kernel changed since
