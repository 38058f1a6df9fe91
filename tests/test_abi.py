"""The C-ABI library loads and exports every entry point include/cmr.h
declares, and rejects bad arguments on the host before touching a GPU.
No call here reaches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

from vlm_decoder_positional_b200 import build as libbuild
from vlm_decoder_positional_b200 import cmr

HEADER = os.path.join(libbuild.INCLUDE, "cmr.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return cmr.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"CMR_API\s+[\w\s\*]+?\b(cmr_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert set(names) == {"cmr_positions", "cmr_positions_chunk", "cmr_positions_step",
                          "cmr_rotate_qk", "cmr_positions_rotate_qk",
                          "cmr_positions_rotate_qk_host", "cmr_rotate_qk_shift",
                          "cmr_rotate_qk_cache", "cmr_rotate_qk_kernel",
                          "cmr_rotate_qk_cache_kernel", "cmr_copy_rotated_dims",
                          "cmr_status_string", "cmr_last_error_message",
                          "cmr_last_rotate_kernel", "cmr_version", "cmr_positions_frames",
                          "cmr_positions_frames_workspace_bytes",
                          "cmr_positions_frames_noalloc"}
    assert set(names) == set(cmr.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", libbuild.LIB], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    ours = {s for s in exported if s.startswith("cmr") or "cmr" in s.lower()}
    assert ours == set(declared_functions())


def test_status_strings_and_version(lib):
    for code in (0, 1, 2, 3):
        assert lib.cmr_status_string(code)
    assert b"unknown" in lib.cmr_status_string(99)
    assert lib.cmr_version() == 20200
    assert lib.cmr_last_rotate_kernel() == b""  # nothing launched on this thread


SEC = (ctypes.c_int32 * 3)(11, 11, 10)
FAKE = 0x10000  # a 16-byte aligned address; never dereferenced


@pytest.mark.parametrize("kw", [
    dict(n_tokens=-1), dict(num_layers=-1), dict(hq=0, hk=0), dict(hq=-1),
    dict(head_dim=250), dict(rot_dim=24), dict(rot_dim=0), dict(rot_dim=512, head_dim=512),
    dict(rot_dim=128, head_dim=64), dict(theta=0.0), dict(theta=float("inf")),
    dict(theta=float("nan")), dict(sections=(12, 11, 10)), dict(sections=(0, 20, 12)),
    dict(q=FAKE + 2), dict(k=FAKE + 8), dict(q=None), dict(pos=None), dict(sections=None),
])
def test_rotate_rejects_bad_arguments_on_the_host(lib, kw):
    a = dict(q=FAKE, k=FAKE, pos=FAKE, n_tokens=10, num_layers=1, hq=8, hk=2, head_dim=256,
             theta=1e7, sections=(11, 11, 10), rot_dim=64)
    a.update(kw)
    sec = None if a["sections"] is None else (ctypes.c_int32 * 3)(*a["sections"])
    st = lib.cmr_rotate_qk(a["q"], a["k"], a["pos"], a["n_tokens"], a["num_layers"], a["hq"],
                           a["hk"], a["head_dim"], a["theta"], sec, a["rot_dim"], None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()
    assert lib.cmr_last_error_message()


def test_rotate_too_many_head_rows_is_unsupported(lib):
    st = lib.cmr_rotate_qk(FAKE, FAKE, FAKE, 10, 80000, 30000, 2, 256, 1e7, SEC, 64, None, None)
    assert st == cmr.CMR_EUNSUPPORTED


def test_rotate_empty_work_is_a_no_op(lib):
    assert lib.cmr_rotate_qk(None, None, None, 0, 1, 8, 2, 256, 1e7, SEC, 64, None, None) == 0
    assert lib.cmr_rotate_qk(None, None, None, 10, 0, 8, 2, 256, 1e7, SEC, 64, None, None) == 0


@pytest.mark.parametrize("args", [
    (FAKE, FAKE, -1, 10), (FAKE, FAKE, 1, -1), (FAKE, FAKE, 0, 10), (FAKE, FAKE, 1, 2 ** 31),
    (FAKE, None, 1, 10), (None, FAKE, 1, 10),
])
def test_positions_rejects_bad_arguments_on_the_host(lib, args):
    ids, cu, b, n = args
    st = lib.cmr_positions(ids, cu, b, n, 248078, FAKE if ids else None, FAKE, FAKE, None, None)
    assert st == cmr.CMR_EINVAL


def test_positions_empty_batch_is_a_no_op(lib):
    assert lib.cmr_positions(None, None, 0, 0, 248078, None, None, None, None, None) == 0
    assert lib.cmr_positions_step(None, None, None, 0, None, None) == 0
    assert lib.cmr_positions_step(None, None, None, -1, None, None) == cmr.CMR_EINVAL


@pytest.mark.parametrize("kw", [
    dict(theta=0.0), dict(rot_dim=24), dict(sections=(12, 11, 10)), dict(hq=0, hk=0),
    dict(num_seqs=-1), dict(num_seqs=0, n_tokens=10), dict(cu=None), dict(q=FAKE + 2),
])
def test_positions_rotate_rejects_bad_arguments_of_either_step(lib, kw):
    # the checks of both steps run before anything is enqueued; with no tokens
    # the rotation's own arguments are still checked
    a = dict(ids=None, cu=None, num_seqs=0, n_tokens=0, q=None, k=None, hq=8, hk=2,
             theta=1e7, sections=(11, 11, 10), rot_dim=64)
    if "cu" in kw or "q" in kw:
        a.update(ids=FAKE, cu=FAKE, num_seqs=1, n_tokens=10, q=FAKE, k=FAKE)
    a.update(kw)
    sec = (ctypes.c_int32 * 3)(*a["sections"])
    st = lib.cmr_positions_rotate_qk(a["ids"], a["cu"], a["num_seqs"], a["n_tokens"], 248078,
                                     FAKE, FAKE, FAKE, a["q"], a["k"], 1, a["hq"], a["hk"], 256,
                                     a["theta"], sec, a["rot_dim"], None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


@pytest.mark.parametrize("kw", [
    dict(grid_side=0), dict(grid_side=129), dict(ws=None), dict(ws_bytes=16 * 3 - 1),
    dict(ws=FAKE + 8), dict(num_seqs=-1), dict(cu=None),
])
def test_positions_frames_rejects_bad_arguments_on_the_host(lib, kw):
    a = dict(ids=FAKE, cu=FAKE, num_seqs=3, n_tokens=30, grid_side=8, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    st = lib.cmr_positions_frames(a["ids"], a["cu"], a["num_seqs"], a["n_tokens"], 248078,
                                  a["grid_side"], FAKE, FAKE, FAKE, a["ws"], a["ws_bytes"], None,
                                  None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


def test_positions_frames_workspace_size():
    # 16 bytes per sequence per slice of about 4,096 tokens
    assert cmr.positions_frames_workspace_bytes(0, 0) == 0
    assert cmr.positions_frames_workspace_bytes(1, 80) == 16
    assert cmr.positions_frames_workspace_bytes(32, 32 * 8192) == 16 * 32 * 2
    assert cmr.positions_frames_workspace_bytes(1, 300_000) == 16 * 74
    assert lib_ok(cmr.lib().cmr_positions_frames(None, None, 0, 0, 248078, 8, None, None, None,
                                                 None, 0, None, None))


def lib_ok(status):
    return status == cmr.CMR_OK


def test_positions_rotate_of_nothing_is_a_no_op(lib):
    assert lib.cmr_positions_rotate_qk(None, None, 0, 0, 248078, None, None, None, None, None, 1,
                                       8, 2, 256, 1e7, SEC, 64, None, None) == 0
    assert lib.cmr_positions_rotate_qk_host(None, None, 0, 0, 248078, None, None, None, None,
                                            None, 1, 8, 2, 256, 1e7, SEC, 64, None, None) == 0


@pytest.mark.parametrize("kw", [dict(theta=0.0), dict(rot_dim=40), dict(head_dim=12),
                                dict(num_seqs=-1), dict(n=-5), dict(cu=None)])
def test_positions_rotate_host_rejects_bad_arguments_on_the_host(lib, kw):
    # refused before anything is enqueued (no GPU needed)
    a = dict(ids=FAKE, cu=FAKE, num_seqs=2, n=10, theta=1e7, rot_dim=64, head_dim=256)
    a.update(kw)
    st = lib.cmr_positions_rotate_qk_host(a["ids"], a["cu"], a["num_seqs"], a["n"], 248078,
                                          FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, a["head_dim"],
                                          a["theta"], SEC, a["rot_dim"], None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


@pytest.mark.parametrize("kw", [
    dict(rule=3), dict(rule=-1), dict(num_seqs=-1), dict(cu=None),
    dict(in_start=FAKE + 64, out_start=FAKE + 64), dict(in_amount=FAKE + 64, out_start=FAKE + 64),
    dict(in_start=FAKE + 60, out_amount=FAKE + 64),
])
def test_positions_chunk_rejects_bad_arguments_on_the_host(lib, kw):
    a = dict(ids=FAKE, cu=FAKE, num_seqs=2, n=10, rule=0, off=None, in_start=FAKE + 256,
             in_amount=FAKE + 512, pos=FAKE, out_start=FAKE + 1024, out_amount=FAKE + 2048)
    a.update(kw)
    st = lib.cmr_positions_chunk(a["ids"], a["cu"], a["num_seqs"], a["n"], 248078, a["rule"],
                                 a["off"], a["in_start"], a["in_amount"], a["pos"],
                                 a["out_start"], a["out_amount"], None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


@pytest.mark.parametrize("kw", [
    dict(num_seqs=0), dict(start=None), dict(amount=None), dict(cu=None, num_seqs=3),
    dict(rot_dim=24), dict(q=FAKE + 4),
])
def test_rotate_shift_rejects_bad_arguments_on_the_host(lib, kw):
    a = dict(q=FAKE, k=FAKE, cu=FAKE, num_seqs=2, off=None, start=FAKE, amount=FAKE, n=10,
             rot_dim=64)
    a.update(kw)
    st = lib.cmr_rotate_qk_shift(a["q"], a["k"], a["cu"], a["num_seqs"], a["off"], a["start"],
                                 a["amount"], a["n"], 1, 8, 2, 256, 1e7, SEC, a["rot_dim"], None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


@pytest.mark.parametrize("kw", [
    dict(v=None), dict(kc=None), dict(vc=None), dict(v=FAKE + 8), dict(kc=FAKE + 4),
    dict(seqs=0), dict(ctx=0), dict(num_seqs=0), dict(start=None),
])
def test_rotate_cache_rejects_bad_arguments_on_the_host(lib, kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, seqs=4, ctx=64, num_seqs=2, start=FAKE)
    a.update(kw)
    st = lib.cmr_rotate_qk_cache(a["q"], a["k"], a["v"], FAKE, a["num_seqs"], None, a["start"],
                                 FAKE, 10, 1, 8, 2, 256, 1e7, SEC, 64, a["kc"], a["vc"],
                                 a["seqs"], a["ctx"], None, None, None)
    assert st == cmr.CMR_EINVAL, lib.cmr_last_error_message()


@pytest.mark.parametrize("args", [
    (FAKE, FAKE, -1, 256, 64, 0), (FAKE, FAKE, 10, 64, 128, 0), (FAKE, FAKE, 10, 256, 64, 2),
    (None, FAKE, 10, 256, 64, 0), (FAKE, None, 10, 256, 64, 1), (FAKE, FAKE, 10, 0, 0, 0),
])
def test_copy_rotated_dims_rejects_bad_arguments(lib, args):
    assert lib.cmr_copy_rotated_dims(*args, None) == cmr.CMR_EINVAL


def test_copy_rotated_dims_of_nothing_is_a_no_op(lib):
    assert lib.cmr_copy_rotated_dims(None, None, 0, 256, 64, 0, None) == cmr.CMR_OK


def test_kernel_query_names_the_path_each_shape_takes(lib):
    def name(*a):
        r = lib.cmr_rotate_qk_kernel(*a)
        return None if r is None else r.decode()
    staged, regs = "rotate_qk_staged_kernel", "rotate_qk_kernel"
    assert name(262144, 6, 8, 2, 256, 64) == staged      # the 6-layer prefill batch
    assert name(262144, 1, 8, 2, 256, 64) == staged
    assert name(8192, 6, 8, 2, 256, 64) == staged        # 1024 tiles of 8 tokens
    assert name(8185, 6, 8, 2, 256, 64) == staged        # 1024 tiles, the last of one token
    assert name(8184, 6, 8, 2, 256, 64) == regs          # 1023 tiles
    assert name(1024, 6, 8, 2, 256, 64) == regs          # a decode step
    assert name(262144, 6, 8, 2, 256, 128) == regs       # rot_dim other than 64
    assert name(262144, 2, 64, 64, 256, 64) == regs      # a stage of 128 head rows is too big
    assert name(262144, 2, 16, 4, 256, 64) == staged
    assert name(262144, 2, 0, 3, 128, 64) == staged
    for bad in [(0, 6, 8, 2, 256, 64), (10, 0, 8, 2, 256, 64), (10, 1, 0, 0, 256, 64),
                (10, 1, 8, 2, 250, 64), (10, 1, 8, 2, 256, 24), (10, 1, 8, 2, 32, 64),
                (10, 80000, 30000, 2, 256, 64), (-1, 1, 8, 2, 256, 64)]:
        assert name(*bad) is None, bad


def test_cache_kernel_query(lib):
    def name(*a):
        r = lib.cmr_rotate_qk_cache_kernel(*a)
        return None if r is None else r.decode()
    staged, regs = "rotate_qk_cache_staged_kernel", "rotate_qk_cache_kernel"
    assert name(262144, 6, 8, 2, 256, 64) == staged
    assert name(8185, 1, 8, 2, 256, 64) == staged
    assert name(8184, 1, 8, 2, 256, 64) == regs
    assert name(1024, 6, 8, 2, 256, 64) == regs           # decode
    assert name(262144, 6, 8, 2, 256, 128) == regs         # rot_dim other than 64
    assert name(262144, 6, 8, 0, 256, 64) == regs          # no K/V: nothing to cache
    assert name(262144, 6, 16, 4, 256, 64) == regs         # 48-KB stage: too big
    assert name(262144, 6, 8, 2, 512, 64) == regs          # head_dim over one box
    assert name(262144, 6, 8, 1, 72, 64) == regs           # 144-B token rows
    assert name(262144, 6, 8, 2, 64, 64) == staged
    assert name(0, 6, 8, 2, 256, 64) is None
