"""The ragged parity cases again, through the bounds-checking build of the library.

``_lib/libkdkl_debug.so`` is the same sources compiled with ``-DKDKL_DEBUG``:
every list walk, partial-result slot, shared-memory list write, TMA coordinate
and lockstep slot in the kernels is range-checked, and a failed check sets
KDKL_DEV_BOUNDS in the device flag word instead of making the access.  A memory
checker is not available on the test machines, so this build stands in for
it.  Each case below is an existing parity test (ragged N, d and V, chunked
backward, every tile width, data errors, variants, the compact cache, the fused
step and the top-K producer); run here, it must still match the oracle, and the
flags it reads must still equal the oracle's data-error flags, which would not
hold if any bounds check had fired.
"""
import pytest

import output_head_kl_b200 as K
from tests import test_gpu_fused_step as FS
from tests import test_gpu_parity as P
from tests import test_gpu_tile_widths as TW
from tests import test_gpu_topk as TK
from tests import test_gpu_variants as VA

pytestmark = pytest.mark.gpu


def _expand(fn):
    """(function, kwargs) for every parameter set of a test (one parametrize mark at most)."""
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    if not marks:
        return [(fn, {})]
    assert len(marks) == 1, fn.__name__
    names, values = marks[0].args[0], marks[0].args[1]
    names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
    out = []
    for v in values:
        v = v.values if hasattr(v, "values") else v
        if len(names) == 1 and not (isinstance(v, tuple) and len(v) == 1):
            v = (v,)
        out.append((fn, dict(zip(names, v))))
    return out


CASES = [c for fn in (
    P.test_tiny_config, P.test_ragged_shapes_multi_tile, P.test_backward_chunks_agree, P.test_grad_loss_scale,
    P.test_temperature_two, P.test_data_errors_flagged_and_handled, P.test_every_row_masked, P.test_empty_batch,
    P.test_one_hot_teacher_is_cross_entropy, P.test_full_teacher_K_equals_V, P.test_largest_cache_K256,
    P.test_ragged_cache_K255_with_duplicates, P.test_minimal_shapes, P.test_single_entry_vocabulary,
    TW.test_every_tile_width_matches_oracle_and_each_other,
    VA.test_compact_cache_matches_oracle_and_wide_cache, VA.test_loss_variants_match_oracle,
    VA.test_variant_with_full_cache_and_label_insertion, VA.test_count_valid_matches_the_oracle_count_and_flags,
    FS.test_ragged_shapes_vs_oracle_and_separate_calls, FS.test_many_chunks_grad_scale_and_data_errors,
    FS.test_variants_and_compact_cache,
    TK.test_topk_matches_oracle_ragged, TK.test_topk_exact_ties_to_smaller_index, TK.test_topk_long_vocabulary_splits,
) for c in _expand(fn)]


# entry points that take a workspace, and the position of the workspace argument
_WS_ARG = {"kdkl_forward": 8, "kdkl_backward": 10, "kdkl_forward_ex": 8, "kdkl_backward_ex": 10,
           "kdkl_forward_backward": 10, "kdkl_teacher_topk": 5, "kdkl_count_valid": 5}


@pytest.fixture
def debug_library(monkeypatch):
    """Every binding call in the test goes to the bounds-checking library, and after every
    call that has a workspace its flag word must not carry KDKL_DEV_BOUNDS."""
    monkeypatch.setattr(K, "LIB_PATH", K.DEBUG_LIB_PATH)
    monkeypatch.setattr(K, "_lib", None)
    lib = K.lib()
    assert lib._name == K.DEBUG_LIB_PATH
    calls = []

    def checked(name, fn, pos):
        def call(*args, **kw):
            st = fn(*args, **kw)
            ws = kw.get("workspace", args[pos] if len(args) > pos else None)
            if st == K.KDKL_OK and ws is not None:
                flags = K.kdkl_read_device_flags(ws)
                assert not flags & K.DEV_BOUNDS, f"{name}: an in-kernel bounds check failed (flags {flags:#x})"
                calls.append(name)
            return st
        return call

    for name, pos in _WS_ARG.items():
        monkeypatch.setattr(K, name, checked(name, getattr(K, name), pos))
    yield calls


@pytest.mark.parametrize("fn,kwargs", CASES,
                         ids=[f"{fn.__module__.split('.')[-1]}.{fn.__name__}{list(kw.values()) or ''}"
                              for fn, kw in CASES])
def test_case_under_bounds_checks(debug_library, fn, kwargs):
    fn(**kwargs)
    assert debug_library, "the case made no call with a workspace"
