"""Sizes the pages work out (tests/golden/page_sizes.json), and what this library needs
at the same shapes.

The pages price the dense approach by its N x V tensors and give the offline cache
format 2 + 2 bytes per entry.  The fixtures pin those formulas to the printed values;
the library's workspace at the pages' shapes must then stay far below a single dense
tensor (it holds no N x V buffer), and its compact cache format is the pages' 4-byte
entry.
"""
import json
import os

import pytest

import output_head_kl_b200 as K

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_sizes.json")


@pytest.fixture(scope="module")
def pages():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def lib():
    from output_head_kl_b200 import build
    build.build()
    return K.lib()


def test_printed_sizes_follow_from_their_parameters(pages):
    p = pages["dense_teacher_probabilities"]
    got = p["batch"] * p["seq_len"] * p["vocab"] * p["bytes_per_value"] / 1e9
    assert abs(got - p["printed_gb"]) <= 0.05 * p["printed_gb"]          # "approximately"
    p = pages["dense_logits_one_tensor"]
    got = p["batch"] * p["seq_len"] * p["vocab"] * p["bytes_per_value"] / 1e9
    assert abs(got - p["printed_gb"]) <= 0.01 * p["printed_gb"]
    p = pages["topk_cache"]
    assert p["tokens"] * p["K"] * (p["bytes_index"] + p["bytes_value"]) / 1e9 == p["printed_gb"]


def test_workspace_far_below_one_dense_tensor(pages, lib):
    # the 8B-class head at the note's shape: 8 x 4096 tokens, d = 4096, K = 100
    p = pages["dense_logits_one_tensor"]
    N, V = p["batch"] * p["seq_len"], p["vocab"]
    dense = N * V * p["bytes_per_value"]
    ws = K.kdkl_workspace_bytes(N, 4096, V, 100)
    assert 0 < ws < 0.3 * dense
    # doubling the tokens adds per-token lists only (no vocabulary-sized term)
    per_token = (K.kdkl_workspace_bytes(2 * N, 4096, V, 100) - ws) / N
    assert per_token < 1024 < 2 * V
    # the article's gpt-oss example: 4 x 32000 tokens over 201,088 entries (d = 2880)
    p = pages["dense_teacher_probabilities"]
    N, V = p["batch"] * p["seq_len"], p["vocab"]
    assert K.kdkl_workspace_bytes(N, 2880, V, 100) < 0.1 * N * V * p["bytes_per_value"]


def test_compact_cache_is_the_pages_entry_format(pages, lib):
    p = pages["topk_cache"]
    # KDKL_CACHE_U16_BF16: uint16 index + bf16 logit per cached entry
    assert p["bytes_index"] + p["bytes_value"] == 2 + 2
    # the note: 16-bit indices suffice while the vocabulary fits them; the library refuses
    # a larger vocabulary on the host, before it touches a device (the placeholder
    # pointers are never dereferenced: only calls that a host check refuses are made)
    import ctypes
    opts = K.kdkl_options(cache_format=K.CACHE_U16_BF16)
    args = (0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 256, 64)
    big = lib.kdkl_forward_ex(*args, 65537, 8, 1.0, ctypes.byref(opts), 0x60000, 0x70000, 0x80000, 1 << 40, None)
    assert big == 2 and "65536" in K.kdkl_last_error()
