"""The DRAM-traffic record's source digest: comments and layout do not change it, code does."""
import os

import bench

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "output_head_kl_b200", "csrc")


def _reader(edit=None):
    def read(name):
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            text = f.read()
        return edit(name, text) if edit else text
    return read


def test_digest_ignores_comments_and_layout():
    base = bench.kernel_sources_digest()
    assert bench.kernel_sources_digest(_reader()) == base

    def recomment(name, text):
        if name != "kernels.cu":
            return text
        return "// a new leading comment\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 5)
    assert bench.kernel_sources_digest(_reader(recomment)) == base


def test_digest_sees_code_changes():
    base = bench.kernel_sources_digest()

    def retune(name, text):
        if name != "kdkl_internal.h":
            return text
        assert "constexpr int kTopKMax = 128;" in text
        return text.replace("constexpr int kTopKMax = 128;", "constexpr int kTopKMax = 96;")
    assert bench.kernel_sources_digest(_reader(retune)) != base


def test_committed_record_is_complete():
    rec = bench.json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert len(rec["sources_sha256"]) == 64
    for wl in ("8b", "large_vocab"):
        assert set(rec["workloads"][wl]) == {"fwd_lse_gemm", "bwd_grad_gemm", "bwd_dhidden_gemm", "bwd_dw_gemm"}
