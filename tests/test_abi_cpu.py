"""The C-ABI library on the CPU: it loads, exports every declared symbol and
checks its arguments on the host (no kernel runs here)."""
import ctypes
import os
import re

import pytest

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200 import build, sda, synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return sda.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "sda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sda_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 14
    assert sorted(sda.EXPORTS) == names
    for n in names:
        assert getattr(L, n) is not None


def test_version_and_errors(L):
    assert "sm_100a" in sda.sda_version()
    for code in range(-8, 1):
        assert L.sda_error_string(code)


@pytest.mark.parametrize("w", [S.TINY, S.WAN13B_480P, S.WAN14B_480P, S.WAN14B_720P] + S.sweep_points()[::7],
                         ids=lambda w: w.name)
def test_keep_count_matches_oracle(L, w):
    p = sda.params_of(w)
    assert sda.sda_keep_count(p) == O.keep_count(w.n_kblk, w.sparsity)
    assert sda.sda_workspace_size(p) > 0


def test_keep_counts_of_named_layers(L):
    assert [sda.sda_keep_count(sda.params_of(w)) for w in (S.TINY, S.WAN13B_480P, S.WAN14B_480P, S.WAN14B_720P)] \
        == [8, 52, 26, 36]


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, -4), ("block_k", 128, -4), ("block_q", 32, -4), ("rank", 24, -4), ("L", 2047, -3),
    ("pairs_t", 3, -3), ("sparsity", 1.0, -3), ("sparsity", -0.1, -3), ("rope_base", 0.0, -3),
    ("gate_per_head", 2, -3), ("B", 0, -3), ("causal_frames", -1, -3), ("causal_frames", 3, -3)])
def test_bad_params_rejected_on_host(L, field, value, code):
    p = sda.params_of(S.TINY)
    setattr(p, field, value)
    assert L.sda_keep_count(ctypes.byref(p)) == code
    assert L.sda_workspace_size(ctypes.byref(p)) == 0
    assert L.sda_forward(ctypes.byref(p), *([None] * 8), None, 0, None) == code
    assert L.sda_last_error_detail()


def test_selector_capacity_limit(L):
    """The selector keeps a row of N_kblk scores in registers: 2048 key blocks (131,072 tokens) at most."""
    at_limit = S.TINY.replace(grid_t=1, grid_h=1, grid_w=64 * 2048, B=1, H=1)
    assert L.sda_keep_count(ctypes.byref(sda.params_of(at_limit))) > 0
    past = S.TINY.replace(grid_t=1, grid_h=1, grid_w=64 * 2048 + 1, B=1, H=1)
    assert L.sda_keep_count(ctypes.byref(sda.params_of(past))) == -4
    assert b"2048" in L.sda_last_error_detail()


def test_workspace_checks_before_device(L):
    p = sda.params_of(S.TINY)
    need = sda.sda_workspace_size(p)
    # too small, misaligned, NULL: rejected on the host before any CUDA call
    assert L.sda_block_select(ctypes.byref(p), 16, 16, 16, 256, need - 1, None) == -5
    assert L.sda_block_select(ctypes.byref(p), 16, 16, 16, 128, need, None) == -2
    assert L.sda_block_select(ctypes.byref(p), 16, 16, 16, None, need, None) == -1


def test_host_buffer_size(L):
    p = sda.params_of(S.TINY)
    tensor = 1 * 2048 * 2 * 64 * 2
    assert sda.sda_forward_host_buffer_size(p) >= sda.sda_workspace_size(p) + 4 * tensor


def test_quant_fp8_row_limit(L):
    """sda_quant_fp8 holds a token's H*d channels in one warp's registers: 16384 at most."""
    p = sda.params_of(S.TINY.replace(H=257, d=64))   # 16448 channels per token
    assert L.sda_quant_fp8(ctypes.byref(p), 16, 16, 16, None) == -4
    assert b"16384" in L.sda_last_error_detail()


@pytest.mark.parametrize("w", [S.TINY.replace(causal_frames=1), S.TINY.replace(causal_frames=2),
                               S.WAN14B_720P.replace(causal_frames=3), S.WAN14B_480P.replace(causal_frames=1),
                               S.TINY.replace(grid_t=6, grid_h=7, grid_w=11, block_q=128, causal_frames=2)],
                         ids=lambda w: f"{w.name}-F{w.causal_frames}")
def test_causal_geometry_on_host(L, w):
    """Query blocks tile each chunk on their own; the row width stays the
    last chunk's keep count; the workspace grows by the per-chunk states."""
    p = sda.params_of(w)
    qb = O.causal_query_blocks(w.L, w.chunk_tokens, w.block_q)
    assert sda.sda_query_blocks(p) == w.n_qblk == len(qb)
    assert sda.sda_keep_count(p) == O.keep_count(w.n_kblk, w.sparsity)
    bidir = sda.params_of(w.replace(causal_frames=0))
    assert sda.sda_query_blocks(bidir) == -(-w.L // w.block_q)
    assert sda.sda_workspace_size(p) > 0


def test_causal_frames_must_divide_the_frames(L):
    p = sda.params_of(S.WAN14B_720P.replace(causal_frames=4))   # 21 frames
    assert L.sda_query_blocks(ctypes.byref(p)) == -3
    assert b"causal_frames" in L.sda_last_error_detail()


def test_backward_checks_on_host(L):
    p = sda.params_of(S.TINY)
    need = sda.sda_backward_workspace_size(p)
    assert need > sda.sda_workspace_size(p)
    args = [None] * 15
    assert L.sda_backward(ctypes.byref(p), *args[:14], None, need, None) == -1       # NULL workspace
    assert L.sda_backward(ctypes.byref(p), *args[:14], 256, need - 1, None) == -5    # workspace too small
    assert L.sda_backward(ctypes.byref(p), *args[:14], 256, need, None) == -1        # NULL inputs
    # a causal window takes more scratch (one dC and one suffix sum per chunk) and the same checks
    causal = sda.params_of(S.TINY.replace(causal_frames=1))
    need_c = L.sda_backward_workspace_size(ctypes.byref(causal))
    assert need_c > need
    assert L.sda_backward(ctypes.byref(causal), *args[:14], 256, need_c - 1, None) == -5
    assert L.sda_backward(ctypes.byref(causal), *args[:14], 256, need_c, None) == -1


def test_missing_library_fails_loudly(monkeypatch):
    """Without the built library every call raises: there is no fallback path."""
    monkeypatch.setattr(sda, "LIB_PATH", os.path.join(ROOT, "no-such-dir", "libsda.so"))
    monkeypatch.setattr(sda, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        sda.lib()
    w = S.TINY
    with pytest.raises(RuntimeError, match="no fallback"):
        sda.sda_keep_count(sda.params_of(w))
    with pytest.raises(RuntimeError, match="no fallback"):
        sda.sda_forward(sda.params_of(w), *([None] * 9), 0)
