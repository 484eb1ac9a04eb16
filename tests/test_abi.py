"""The C ABI library on a machine without a GPU: it loads, exports every symbol
that include/*.h declares, and its host-only entry points (validation,
workspace sizing, index maps) behave as documented.  No compute call is made."""
import glob
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle
from structured_attention_video_b200 import _lib, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        names |= set(re.findall(r"MONARCH_API\s+[\w\s\*]+?\b(monarch_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (monarch_\w+)", out))
    assert names <= exported, names - exported
    for name in names:
        assert hasattr(_lib._lib, name)
        assert name in _lib.SIGNATURES


SHAPE_720P = (1, 12, 21, 45, 80, 128, 945, 80, 4, 1)


def test_workspace_bytes_and_validation():
    bf16 = _lib.BF16
    assert _lib.monarch_attn_workspace_bytes(*SHAPE_720P, bf16) > 0
    bad = [
        (1, 12, 21, 45, 80, 128, 944, 80, 4, 1),   # b1*b2 != N
        (1, 12, 21, 45, 80, 128, 945, 80, 0, 1),   # tiles < 1
        (1, 12, 21, 45, 80, 128, 945, 80, 946, 1), # tiles > b1
        (1, 12, 21, 45, 80, 128, 945, 80, 4, 0),   # iters < 1
        (1, 12, 21, 45, 80, 96, 945, 80, 4, 1),    # unsupported d
        (0, 12, 21, 45, 80, 128, 945, 80, 4, 1),   # B < 1
    ]
    for shape in bad:
        assert _lib.monarch_attn_workspace_bytes(*shape, bf16) == 0
        assert _lib.monarch_attn_path(*shape, bf16) == -1
    assert _lib.monarch_attn_workspace_bytes(*SHAPE_720P, 7) == 0


@pytest.mark.parametrize("shape,code", [
    ((1, 2, 3, 8, 8, 32, 25, 8, 1, 1), 2),
    ((1, 2, 3, 8, 8, 32, 24, 8, 25, 1), 2),
    ((1, 2, 3, 8, 8, 48, 24, 8, 1, 1), 4),
    ((1, 0, 3, 8, 8, 32, 24, 8, 1, 1), 1),
])
def test_fwd_rejects_bad_arguments_before_touching_the_device(shape, code):
    fake = 1 << 20   # never dereferenced: validation fails first
    st = _lib.monarch_attn_fwd_ws(fake, fake, fake, fake, *shape, _lib.F32, fake, 1 << 30, None)
    assert st == code
    assert _lib.monarch_attn_fwd(fake, fake, fake, fake, *shape, _lib.F32, None) == code


def test_fwd_rejects_null_and_misaligned_pointers():
    shape = (1, 2, 3, 8, 8, 32, 24, 8, 1, 1)
    fake = 1 << 20
    assert _lib.monarch_attn_fwd_ws(None, fake, fake, fake, *shape, 0, fake, 1 << 30, None) == 1
    assert _lib.monarch_attn_fwd_ws(fake, fake, fake, fake, *shape, 0, None, 1 << 30, None) == 1
    assert _lib.monarch_attn_fwd_ws(fake + 4, fake, fake, fake, *shape, 0, fake, 1 << 30,
                                    None) == 3
    assert _lib.monarch_attn_fwd_ws(fake, fake, fake, fake, *shape, 0, fake + 64, 1 << 30,
                                    None) == 3
    assert _lib.monarch_attn_fwd_ws(fake, fake, fake, fake, *shape, 0, fake, 16, None) == 5
    assert _lib.monarch_attn_fwd_host(None, fake, fake, fake, *shape, 0, None) == 1


def test_profile_kernel_names():
    """Every kernel family has a distinct name, and out-of-range ids return NULL."""
    names = []
    k = 0
    while _lib.monarch_profile_kernel_name(k) is not None:
        names.append(_lib.monarch_profile_kernel_name(k))
        k += 1
    assert len(names) == len(set(names)) == 16
    assert _lib.monarch_profile_kernel_name(-1) is None
    for name in ("tc_lstep_kernel", "tc_rstep_kernel", "tc_qbar_kernel", "tc_bwd_dq_kernel<0>",
                 "tc_bwd_dkz_kernel", "tc_bwd_dq_kernel<1>", "tc_bwd_r_kernel"):
        assert name in names


def test_status_strings():
    for code in range(8):
        assert len(_lib.monarch_status_string(code)) > 0
    assert _lib.monarch_status_string(99) == "unknown status"


@pytest.mark.parametrize("f,h,w,b1,b2,tiles", [(3, 8, 8, 24, 8, 1), (3, 8, 8, 24, 8, 5),
                                                (3, 8, 8, 1, 192, 1), (3, 8, 8, 192, 1, 192),
                                                (3, 30, 52, 90, 52, 1), (21, 45, 80, 945, 80, 4),
                                                (21, 30, 52, 630, 52, 8)])
def test_host_index_maps_match_oracle_bit_exactly(f, h, w, b1, b2, tiles):
    N = f * h * w
    u, v, p = (np.full(N, -1, np.int32) for _ in range(3))
    t = np.full(tiles + 1, -1, np.int32)
    assert _lib.monarch_index_maps(f, h, w, b1, b2, tiles, u, v, p, t) == 0
    ref = oracle.index_maps(f, h, w, b1, b2, tiles)
    assert np.array_equal(u, ref["u_of_n"])
    assert np.array_equal(v, ref["v_of_n"])
    assert np.array_equal(p, ref["perm"])
    assert np.array_equal(t, ref["tile_lo"])
    assert _lib.monarch_index_maps(f, h, w, b1 + 1, b2, tiles, u, v, p, t) == 2


def test_workspace_covers_intermediates():
    """Enough room for Ktil and Z of every (head, tile, column, block) at least in bf16."""
    wl = synth.WORKLOADS["720p"]
    need = _lib.monarch_attn_workspace_bytes(*SHAPE_720P, _lib.BF16)
    assert need >= 2 * wl.B * wl.H * wl.tiles * wl.N * wl.d * 2


def test_backward_workspace_and_validation():
    """The backward's workspace: 0 for iters != 1 or a failing shape; otherwise at
    least the forward's intermediates plus the backward's float32 arrays; the
    calls reject bad arguments before touching the device."""
    shape = (1, 2, 3, 8, 8, 32, 24, 8, 5)   # B, H, f, h, w, d, b1, b2, tiles
    fw = _lib.monarch_attn_workspace_bytes(*shape, 1, _lib.F32)
    bw = _lib.monarch_attn_bwd_workspace_bytes(*shape, 1, _lib.F32)
    B, H, N, d, t = 1, 2, 192, 32, 5
    floats = (2 * B * H * N + B * H * N * d + 2 * B * H * t * N * d + 4 * B * H * t * N)
    assert bw >= fw + 4 * floats
    assert _lib.monarch_attn_bwd_workspace_bytes(*shape, 2, _lib.F32) == 0
    assert _lib.monarch_attn_bwd_workspace_bytes(1, 2, 3, 8, 8, 32, 25, 8, 5, 1, _lib.F32) == 0
    # iters = 2: refused before anything is enqueued
    assert _lib.monarch_attn_bwd(16, 16, 16, 16, 16, 16, 16, *shape, 2, _lib.F32,
                                 None) == 4   # MONARCH_ERR_UNSUPPORTED
    # a null gradient pointer
    assert _lib.monarch_attn_bwd_ws(16, 16, 16, 16, None, 16, 16, *shape, 1, _lib.F32, 256,
                                    bw, None) == 1   # MONARCH_ERR_INVALID_ARG


def test_tiled_entry_points_validate_the_axis_and_tile_range():
    """Key-column tiles take tiles in [1, b2] and the generic kernels; the
    query-row axis is the default entry points' reading, bit for bit the same
    workspace; a bad axis or range is refused before touching the device."""
    shape = (1, 2, 3, 8, 8, 32, 24, 8)          # B, H, f, h, w, d, b1, b2
    Q, K = _lib.TILE_QUERY_ROWS, _lib.TILE_KEY_COLUMNS
    for t in (1, 5, 24):
        assert (_lib.monarch_attn_tiled_workspace_bytes(*shape, t, 1, _lib.F32, Q) ==
                _lib.monarch_attn_workspace_bytes(*shape, t, 1, _lib.F32))
    for t in (1, 3, 8):
        assert _lib.monarch_attn_tiled_workspace_bytes(*shape, t, 2, _lib.F32, K) > 0
        assert _lib.monarch_attn_tiled_path(*shape, t, 1, _lib.BF16, K) == 0
    assert _lib.monarch_attn_tiled_workspace_bytes(*shape, 9, 1, _lib.F32, K) == 0   # t > b2
    assert _lib.monarch_attn_tiled_workspace_bytes(*shape, 0, 1, _lib.F32, K) == 0
    assert _lib.monarch_attn_tiled_workspace_bytes(*shape, 2, 1, _lib.F32, 2) == 0   # bad axis
    assert _lib.monarch_attn_tiled_path(*shape, 9, 1, _lib.F32, K) == -1
    ws = _lib.monarch_attn_tiled_workspace_bytes(*shape, 3, 1, _lib.F32, K)
    assert _lib.monarch_attn_fwd_tiled_ws(16, 16, 16, 16, *shape, 9, 1, _lib.F32, K, _lib.BHND,
                                          256, ws, None) == 2          # MONARCH_ERR_SHAPE
    assert _lib.monarch_attn_fwd_tiled_ws(16, 16, 16, 16, *shape, 3, 1, _lib.F32, 7, _lib.BHND,
                                          256, ws, None) == 1          # bad axis
    assert _lib.monarch_attn_fwd_tiled_ws(16, 16, 16, 16, *shape, 3, 1, _lib.F32, K, 5,
                                          256, ws, None) == 1          # bad layout
    assert _lib.monarch_attn_fwd_tiled_ws(16, 16, 16, 16, *shape, 3, 1, _lib.F32, K, _lib.BHND,
                                          256, ws - 1, None) == 5      # workspace too small
    assert _lib.monarch_attn_fwd_tiled_ws(16, 16, 16, 24, *shape, 3, 1, _lib.F32, K, _lib.BHND,
                                          256, ws, None) == 3          # misaligned out
