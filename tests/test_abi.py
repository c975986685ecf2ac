"""The C ABI without a GPU: the library loads, exports what include/mla.h declares,
and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]*?\b(mla_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from deepseek_mla_latent_b200 import build
    build.build()
    from deepseek_mla_latent_b200 import _lib
    return _lib


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("mla_absorb_q", "mla_attn_decode", "mla_attn_prefill_chunk", "mla_out_proj",
                     "mla_workspace_size", "mla_status_string", "mla_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert names
    for n in names:
        assert hasattr(lib.LIB, n), n
        assert n in lib.SIGNATURES, f"binding lacks {n}"


def test_version_and_status_strings(lib):
    assert lib.LIB.mla_api_version() == 1
    for s in range(6):
        assert lib.LIB.mla_status_string(s)


V3 = dict(heads=128, kv_lora_rank=512, qk_nope=128, qk_rope=64, v_head=128)


def test_kernel_family_selection(lib):
    d = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    assert lib.LIB.mla_kernel_family(ctypes.byref(d)) in (0, 1)
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    assert lib.LIB.mla_kernel_family(ctypes.byref(d)) == 0
    d = lib.make_dims(8, 4096, 32, 16, 32, "f32", 0.1)
    assert lib.LIB.mla_kernel_family(ctypes.byref(d)) == -1
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    d.dtype = 7
    assert lib.LIB.mla_kernel_family(ctypes.byref(d)) == -1


# Fake but aligned device addresses: every call below must return before touching them.
A = 0x10000


def test_host_validation_rejects_before_launch(lib):
    L = lib.LIB
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    bad = lib.make_dims(8, 4096, 32, 16, 32, "f32", 0.1)
    assert L.mla_absorb_q(None, A, 384, A, A, 4, None) == lib.MLA_ERR_INVALID_ARG
    assert L.mla_absorb_q(ctypes.byref(bad), A, 384, A, A, 4, None) == lib.MLA_ERR_UNSUPPORTED
    assert L.mla_absorb_q(ctypes.byref(d), A, 100, A, A, 4, None) == lib.MLA_ERR_INVALID_ARG   # stride < H*(Dn+R)
    assert L.mla_absorb_q(ctypes.byref(d), None, 384, A, A, 4, None) == lib.MLA_ERR_INVALID_ARG
    assert L.mla_absorb_q(ctypes.byref(d), A + 4, 384, A, A, 4, None) == lib.MLA_ERR_INVALID_ARG  # misaligned
    assert L.mla_absorb_q(ctypes.byref(d), A, 384, A, A, -1, None) == lib.MLA_ERR_INVALID_ARG
    assert L.mla_absorb_q(ctypes.byref(d), None, 384, None, None, 0, None) == lib.MLA_OK        # empty
    assert L.mla_out_proj(ctypes.byref(d), A, None, A, 3, None) == lib.MLA_ERR_INVALID_ARG
    assert L.mla_out_proj(ctypes.byref(d), None, None, None, 0, None) == lib.MLA_OK
    # decode: too many splits, negative batch, missing cache
    assert L.mla_attn_decode(ctypes.byref(d), A, A, 384, A, A, 256, A, 2, 128, A, A, 1 << 20, 300, None) \
        == lib.MLA_ERR_INVALID_ARG
    assert L.mla_attn_decode(ctypes.byref(d), A, A, 384, A, A, 256, A, -1, 128, A, A, 1 << 20, 0, None) \
        == lib.MLA_ERR_INVALID_ARG
    assert L.mla_attn_decode(ctypes.byref(d), A, A, 384, None, A, 256, A, 2, 128, A, A, 1 << 20, 0, None) \
        == lib.MLA_ERR_INVALID_ARG
    assert L.mla_attn_decode(ctypes.byref(d), None, None, 384, None, None, 0, None, 0, 0, None, None, 0, 0, None) \
        == lib.MLA_OK
    # prefill: missing cu_seqlens_q
    assert L.mla_attn_prefill_chunk(ctypes.byref(d), A, A, 384, None, A, 2, 8, 4, 128, A, A, 256, A, A, 1 << 20,
                                    None) == lib.MLA_ERR_INVALID_ARG


def test_workspace_is_checked(lib):
    L = lib.LIB
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    need = L.mla_workspace_size(ctypes.byref(d), 2, 2, 1 << 16, 4)
    assert need > 0
    assert L.mla_attn_decode(ctypes.byref(d), A, A, 384, A, A, 1 << 17, A, 2, 1 << 16, A, A, need - 16, 4, None) \
        == lib.MLA_ERR_WORKSPACE
    assert L.mla_attn_decode(ctypes.byref(d), A, A, 384, A, A, 1 << 17, A, 2, 1 << 16, A, None, need, 4, None) \
        == lib.MLA_ERR_WORKSPACE
    assert L.mla_workspace_size(ctypes.byref(d), 2, 2, 1 << 16, 1) == 0
    v3 = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    assert L.mla_workspace_size(ctypes.byref(v3), 8, 8, 4096, 0) >= 0


def test_decode_out_host_checks(lib):
    L = lib.LIB
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    need = L.mla_decode_out_workspace_size(ctypes.byref(d), 2, 1 << 16, 4)
    # o_lat [2, 8, 64] fp32 plus the split partials of the attention call
    assert need >= 2 * 8 * 64 * 4 + L.mla_workspace_size(ctypes.byref(d), 2, 2, 1 << 16, 4)
    args = lambda ws, wsb, wkv_b=A: (ctypes.byref(d), A, A, 384, A, A, 1 << 17, A, 2, 1 << 16, wkv_b, A, ws, wsb, 4, None)
    assert L.mla_attn_decode_out(*args(A, need - 16)) == lib.MLA_ERR_WORKSPACE
    assert L.mla_attn_decode_out(*args(None, need)) == lib.MLA_ERR_WORKSPACE
    assert L.mla_attn_decode_out(*args(A, need, wkv_b=None)) == lib.MLA_ERR_INVALID_ARG
    assert L.mla_attn_decode_out(ctypes.byref(d), None, None, 384, None, None, 0, None, 0, 0, None, None, None, 0, 0,
                                 None) == lib.MLA_OK
    assert L.mla_decode_out_workspace_size(ctypes.byref(d), 2, 1 << 16, 300) == 0


def test_append_host_checks(lib):
    L = lib.LIB
    v3 = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    f = lambda *a: L.mla_append_latent(ctypes.byref(v3), *a)
    assert f(A, A, None, 1e-6, 10000.0, A, A, 0, None, None, 0, None) == lib.MLA_OK            # nothing to write
    assert f(A, A, None, 1e-6, 10000.0, A, A, -1, A, A, 8, None) == lib.MLA_ERR_INVALID_ARG    # negative count
    assert f(A, A, None, -1.0, 10000.0, A, A, 4, A, A, 8, None) == lib.MLA_ERR_INVALID_ARG     # eps < 0
    assert f(A, A, None, 1e-6, 0.0, A, A, 4, A, A, 8, None) == lib.MLA_ERR_INVALID_ARG         # base <= 0
    assert f(A, A, None, 1e-6, 10000.0, None, A, 4, A, A, 8, None) == lib.MLA_ERR_INVALID_ARG  # no positions
    assert f(A + 8, A, None, 1e-6, 10000.0, A, A, 4, A, A, 8, None) == lib.MLA_ERR_INVALID_ARG  # misaligned
    odd = lib.make_dims(128, 500, 128, 64, 128, "bf16", 0.07)   # C not a multiple of 8
    assert L.mla_append_latent(ctypes.byref(odd), A, A, None, 1e-6, 10000.0, A, A, 4, A, A, 8, None) \
        == lib.MLA_ERR_UNSUPPORTED


def test_paged_host_checks(lib):
    L = lib.LIB
    d = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    v3 = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    need = L.mla_workspace_size(ctypes.byref(d), 2, 2, 1 << 12, 4)

    def call(dims=d, cu_q=None, n_q=2, seqlens=A, batch=2, num_pages=64, page=64, table=A, stride=64,
             ws=A, wsb=need, splits=4):
        return L.mla_attn_paged(ctypes.byref(dims), A, A, 384, cu_q, n_q, seqlens, batch, 1 << 12, A, A, num_pages,
                                page, table, stride, A, ws, wsb, splits, None)

    assert call(batch=0, n_q=0) == lib.MLA_OK
    assert call(page=0) == lib.MLA_ERR_INVALID_ARG
    assert call(num_pages=-1) == lib.MLA_ERR_INVALID_ARG
    assert call(stride=-1) == lib.MLA_ERR_INVALID_ARG
    assert call(table=None) == lib.MLA_ERR_INVALID_ARG
    assert call(seqlens=None) == lib.MLA_ERR_INVALID_ARG
    assert call(n_q=3) == lib.MLA_ERR_INVALID_ARG                 # decode has one query per sequence
    assert call(cu_q=A, n_q=5, splits=4) == lib.MLA_ERR_INVALID_ARG  # prefill takes no splits
    assert call(ws=None) == lib.MLA_ERR_WORKSPACE
    assert call(wsb=need - 16) == lib.MLA_ERR_WORKSPACE
    # the tensor-core kernels copy 64-key tiles: smaller pages are not built for them
    assert L.mla_attn_paged(ctypes.byref(v3), A, A, 128 * 192, None, 2, A, 2, 1 << 12, A, A, 64, 32, A, 128, A,
                            A, 1 << 30, 0, None) == lib.MLA_ERR_UNSUPPORTED


def test_expand_host_checks(lib):
    L = lib.LIB
    v3 = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    f = lambda *a: L.mla_expand_kv(ctypes.byref(v3), *a)
    assert f(A, None, 1e-6, A, 0, 128, A, A, None) == lib.MLA_OK              # no tokens
    assert f(A, None, 1e-6, A, -1, 128, A, A, None) == lib.MLA_ERR_INVALID_ARG
    assert f(A, None, -1.0, A, 1, 128, A, A, None) == lib.MLA_ERR_INVALID_ARG   # eps < 0
    assert f(None, None, 1e-6, A, 1, 128, A, A, None) == lib.MLA_ERR_INVALID_ARG
    assert f(A, A + 8, 1e-6, A, 1, 128, A, A, None) == lib.MLA_ERR_INVALID_ARG  # misaligned gain
    assert f(A, None, 1e-6, A, 1 << 30, 1 << 30, A, A, None) == lib.MLA_ERR_INVALID_ARG   # token count overflows


@pytest.mark.parametrize("batch", [1, 2, 8, 37, 64, 74, 75, 300])
@pytest.mark.parametrize("max_k", [1, 128, 129, 4096, 131072])
def test_decode_split_plan(lib, batch, max_k):
    """The automatic split plan of the tensor-core decode: at least one split, never more
    splits than 128-key score tiles, no split left empty by the tile rounding, and with more
    than one split no more (row, split) units than CTA pairs of a 148-SM GPU (the host has no
    device here, so the planner uses 148).
    An explicit split count is used as given, and the workspace grows with the splits."""
    L = lib.LIB
    v3 = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    s = L.mla_decode_num_splits(ctypes.byref(v3), batch, max_k, 0)
    tiles = -(-max_k // 128)
    assert 1 <= s <= max(1, tiles)
    if s > 1:
        assert batch * s <= 74
    # splits are whole 128-key tiles; the plan leaves none of them empty for the longest sequence
    per = -(-(-(-max_k // s)) // 128) * 128
    assert -(-max_k // per) == s
    assert L.mla_decode_num_splits(ctypes.byref(v3), batch, max_k, 5) == 5
    w1 = L.mla_workspace_size(ctypes.byref(v3), batch, batch, max_k, 1)
    w2 = L.mla_workspace_size(ctypes.byref(v3), batch, batch, max_k, 2)
    w9 = L.mla_workspace_size(ctypes.byref(v3), batch, batch, max_k, 9)
    assert w1 <= w2 < w9
    # the partials alone: bf16 [splits, batch, H, 512]
    assert w9 >= 9 * batch * 128 * 512 * 2
    out = L.mla_decode_out_workspace_size(ctypes.byref(v3), batch, max_k, 9)
    assert out >= w9 + batch * 128 * 512 * 2


def test_merge_entry_points_host_checks(lib):
    """mla_merge_partials(_out): tensor-core dims only, 1..256 splits, aligned non-null pointers,
    grids that fit; every refusal comes back before any launch (no device here)."""
    d = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    if lib.LIB.mla_kernel_family(ctypes.byref(d)) != 1:
        pytest.skip("tensor-core family not selected")
    L, D = lib.LIB, ctypes.byref(d)
    bad = lib.MLA_ERR_INVALID_ARG
    for f in (lambda *a: L.mla_merge_partials(D, *a[:4], A, None),
              lambda *a: L.mla_merge_partials_out(D, *a[:4], A, A, None)):
        assert f(A, A, 2, 0) == lib.MLA_OK                     # no rows: nothing to do
        assert f(A, A, 0, 8) == bad and f(A, A, 257, 8) == bad  # split count
        assert f(None, A, 2, 8) == bad and f(A, None, 2, 8) == bad
        assert f(A + 8, A, 2, 8) == bad                          # misaligned partials
        assert f(A, A, 2, -1) == bad and f(A, A, 2, 1 << 31) == bad
    assert L.mla_merge_partials(D, A, A, 2, 8, None, None) == bad
    assert L.mla_merge_partials(D, A, A, 2, 1 << 30, A, None) == bad          # grid of (row, head) pairs
    assert L.mla_merge_partials_out(D, A, A, 2, 8, None, A, None) == bad
    assert L.mla_merge_partials_out(D, A, A, 2, 1 << 21, A, A, None) == bad   # row tiles on the grid's y axis
    f32 = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    assert L.mla_merge_partials(ctypes.byref(f32), A, A, 2, 8, A, None) == lib.MLA_ERR_UNSUPPORTED


def test_partials_entry_point_host_checks(lib):
    """mla_attn_decode_partials exists only on the tensor-core kernels and needs its workspace."""
    d = lib.make_dims(**V3, dtype="bf16", softmax_scale=0.07)
    if lib.LIB.mla_kernel_family(ctypes.byref(d)) != 1:
        pytest.skip("tensor-core family not selected")
    n = lib.LIB.mla_partials_workspace_size(ctypes.byref(d), 8, 4096, 9)
    assert n >= 9 * 8 * 128 * 512 * 2 + 9 * 8 * 128 * 8
    assert lib.LIB.mla_partials_workspace_size(ctypes.byref(d), 8, 4096, 1) >= 8 * 128 * 512 * 2
    f32 = lib.make_dims(8, 64, 32, 16, 32, "f32", 0.1)
    assert lib.LIB.mla_partials_workspace_size(ctypes.byref(f32), 1, 128, 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    st = lib.LIB.mla_attn_decode_partials(ctypes.byref(f32), fake, fake, 56, fake, fake, 128, fake, 1, 128, fake,
                                          1 << 20, 0, None)
    assert st == lib.MLA_ERR_UNSUPPORTED
    # a workspace smaller than the size function reports is refused before any launch
    st = lib.LIB.mla_attn_decode_partials(ctypes.byref(d), fake, fake, 128 * 192, fake, fake, 8 * 4096, fake, 8,
                                          4096, fake, 16, 9, None)
    assert st == lib.MLA_ERR_WORKSPACE


def test_fault_injection_hook_only_in_its_own_build(lib):
    """mla_fault_inject.h's hook is exported by the fault-injection build and by nothing else."""
    from deepseek_mla_latent_b200 import build
    path = build.build(variant="fault_inject")
    text = open(os.path.join(ROOT, "include", "mla_fault_inject.h")).read()
    hooks = re.findall(r"MLA_API\s+[\w\s\*]*?\b(mla_\w+)\s*\(", text)
    assert hooks == ["mla_test_set_fault_plan"]
    variant = ctypes.CDLL(path)
    for n in hooks + _declared_functions():
        assert hasattr(variant, n), n
    for n in hooks:
        assert not hasattr(lib.LIB, n), f"the product library exports {n}"
