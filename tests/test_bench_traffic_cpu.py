"""How bench.py ties a roofline's DRAM traffic to a committed ncu summary (CPU only).

A summary under profiles/ records the traffic of one launch together with the sha256
of the kernel sources it was captured from; bench.py reports that traffic only while
those sources are unchanged, so a figure never outlives the code it describes.
"""
import hashlib
import os
import re

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_tree(tmp_path, sources, profile_files, traffic=123456789):
    csrc = tmp_path / "gated_deltanet_sequence_gdn_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in sources.items():
        (csrc / name).write_text(text)
    hs = hashlib.sha256()
    for f in profile_files:
        hs.update((csrc / f).read_bytes())
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k.md").write_text(
        f"# k\n\ntraffic_bytes_per_launch: {traffic}\n"
        f"source_files: {' '.join(profile_files)}\nsource_sha256: {hs.hexdigest()}\n")
    return csrc


def test_traffic_reported_while_the_listed_sources_are_unchanged(tmp_path, monkeypatch):
    _fake_tree(tmp_path, {"a.cu": "kernel a\n", "b.cuh": "header b\n", "c.cu": "other\n"},
               ["a.cu", "b.cuh"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k") == 123456789.0
    assert bench.kernel_traffic("missing") is None


def test_traffic_dropped_when_a_listed_source_changes(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, {"a.cu": "kernel a\n", "b.cuh": "header b\n"}, ["a.cu", "b.cuh"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "b.cuh").write_text("header b, edited\n")
    assert bench.kernel_traffic("k") is None


def test_a_source_outside_the_list_does_not_matter(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, {"a.cu": "kernel a\n", "host.cu": "host code\n"}, ["a.cu"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "host.cu").write_text("host code, edited\n")
    assert bench.kernel_traffic("k") == 123456789.0


def test_the_hash_covers_the_files_in_their_listed_order(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, {"a.cu": "A\n", "b.cu": "B\n"}, ["a.cu", "b.cu"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = tmp_path / "profiles" / "k.md"
    p.write_text(p.read_text().replace("source_files: a.cu b.cu", "source_files: b.cu a.cu"))
    assert bench.kernel_traffic("k") is None
    assert (csrc / "a.cu").exists()


@pytest.mark.parametrize("name", sorted(f[:-3] for f in os.listdir(os.path.join(ROOT, "profiles"))
                                        if f.endswith(".md")))
def test_committed_summaries_name_existing_sources(name):
    txt = open(os.path.join(ROOT, "profiles", f"{name}.md")).read()
    files = re.search(r"source_files:\s*(.+)", txt)
    if files is None:
        pytest.skip("no source list: a launch list, not a traffic figure")
    csrc = os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "csrc")
    for f in files.group(1).split():
        assert os.path.exists(os.path.join(csrc, f)), f
    assert re.search(r"traffic_bytes_per_launch:\s*[0-9]+", txt)
    assert re.search(r"source_sha256:\s*[0-9a-f]{64}", txt)
