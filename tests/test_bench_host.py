"""Host-side logic of the bench (CPU): the roofline traffic figure is taken
from an ncu summary only while the kernel's sources match the capture."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_line_used_only_for_matching_sources(tmp_path):
    digest = bench.kernel_sources_digest("mlp_block")
    (tmp_path / "k.md").write_text(f"text\n\n```\ntraffic mlp_block 123456 {digest}\n"
                                   f"traffic attn_out 777 0000000000000000\n```\n")
    assert bench.measured_traffic("mlp_block", str(tmp_path)) == {"bytes": 123456,
                                                                   "source": os.path.relpath(str(tmp_path / "k.md"),
                                                                                             ROOT)}
    assert bench.measured_traffic("attn_out", str(tmp_path)) is None  # stale capture
    assert bench.measured_traffic("attn_in", str(tmp_path)) is None  # no capture


def test_digest_depends_on_every_header():
    assert bench.kernel_sources_digest("attn_in") == bench.kernel_sources_digest("mlp_block")  # same headers
    assert bench.kernel_sources_digest("attn_out") != bench.kernel_sources_digest("mlp_block")
