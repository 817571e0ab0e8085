"""The C-ABI library builds, loads and exports what include/pkv.h declares;
host-side argument checks answer with a status before any launch (no GPU is
touched: every call here fails validation first)."""
import ctypes
import subprocess

import pytest

from paged_kv_cache_459_b200 import build as pkv_build

pkv_build.build()
from paged_kv_cache_459_b200 import pkv  # noqa: E402

FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation rejects first


def test_header_symbols_are_exported():
    names = pkv.declared_symbols()
    assert len(names) >= 20 and "pkv_paged_kv_write" in names and "pkv_paged_attention_decode" in names
    out = subprocess.run(["nm", "-D", "--defined-only", pkv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(pkv.lib(), n)
    # nothing else of ours leaks out of the library
    assert all(not s.startswith("_ZN3pkv") for s in exported)


def test_status_strings_and_constants():
    assert pkv.lib().pkv_block_tokens() == 16
    assert pkv.status_string(0) == "ok"
    assert pkv.status_string(pkv.ERR_WORKSPACE).startswith("workspace")
    assert pkv.status_string(99) == "unknown status"
    assert b"sm_100a" in pkv.lib().pkv_version()


def decode(**kw):
    args = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, tables=FAKE, W=8, lens=FAKE, B=2, Hq=4, Hkv=2,
                D=128, NB=64, scale=0.1, variant=0, part=512, ws=None, wsb=0)
    args.update(kw)
    return pkv.lib().pkv_paged_attention_decode_ex(
        args["out"], args["q"], args["kc"], args["vc"], args["tables"], args["W"], args["lens"],
        args["B"], args["Hq"], args["Hkv"], args["D"], args["NB"], args["scale"], args["variant"],
        args["part"], args["ws"], args["wsb"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), pkv.ERR_UNSUPPORTED),
    (dict(D=256), pkv.ERR_UNSUPPORTED),
    (dict(Hq=5, Hkv=2), pkv.ERR_INVALID_ARG),
    (dict(Hkv=0), pkv.ERR_INVALID_ARG),
    (dict(q=None), pkv.ERR_INVALID_ARG),
    (dict(tables=None), pkv.ERR_INVALID_ARG),
    (dict(out=FAKE + 2), pkv.ERR_INVALID_ARG),
    (dict(kc=FAKE + 8), pkv.ERR_INVALID_ARG),
    (dict(W=0), pkv.ERR_INVALID_ARG),
    (dict(NB=0), pkv.ERR_INVALID_ARG),
    (dict(B=-1), pkv.ERR_INVALID_ARG),
    (dict(B=70000), pkv.ERR_INVALID_ARG),
    (dict(scale=float("nan")), pkv.ERR_INVALID_ARG),
    (dict(variant=7), pkv.ERR_INVALID_ARG),
    (dict(part=40), pkv.ERR_INVALID_ARG),
    (dict(NB=1 << 26, Hkv=2), pkv.ERR_UNSUPPORTED),
    (dict(variant=2), pkv.ERR_WORKSPACE),
    (dict(variant=2, ws=FAKE, wsb=16), pkv.ERR_WORKSPACE),
])
def test_decode_argument_checks(kw, code):
    assert decode(**kw) == code


def step(**kw):
    """pkv_paged_decode_step: decode's arguments plus the step's new K and V."""
    args = dict(out=FAKE, q=FAKE, kn=FAKE, vn=FAKE, kc=FAKE, vc=FAKE, tables=FAKE, W=8, lens=FAKE,
                B=2, Hq=4, Hkv=2, D=128, NB=64, scale=0.1, variant=0, part=512, ws=None, wsb=0)
    args.update(kw)
    return pkv.lib().pkv_paged_decode_step(
        args["out"], args["q"], args["kn"], args["vn"], args["kc"], args["vc"], args["tables"],
        args["W"], args["lens"], args["B"], args["Hq"], args["Hkv"], args["D"], args["NB"],
        args["scale"], args["variant"], args["part"], args["ws"], args["wsb"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(kn=None), pkv.ERR_INVALID_ARG),
    (dict(vn=None), pkv.ERR_INVALID_ARG),
    (dict(kn=FAKE + 4), pkv.ERR_INVALID_ARG),
    (dict(D=96), pkv.ERR_UNSUPPORTED),
    (dict(variant=3, ws=FAKE, wsb=1 << 40), pkv.ERR_INVALID_ARG),   # 3 is not a variant
    (dict(variant=2), pkv.ERR_WORKSPACE),
])
def test_fused_step_argument_checks(kw, code):
    assert step(**kw) == code


def test_fused_step_empty_batch_is_a_no_op():
    assert step(B=0, out=None, q=None, kn=None, vn=None) == pkv.OK


def test_cascade_steps_check_their_arguments():
    L = pkv.lib()
    common = (FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 2, 4, 2, 128, 64, 0.1, FAKE, FAKE, FAKE, 1)
    # fused: a missing new K
    assert L.pkv_paged_decode_prefix_step(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 2, 4, 2,
                                          128, 64, 0.1, FAKE, FAKE, FAKE, 1, 0, 512, FAKE, 1 << 30,
                                          None, None) == pkv.ERR_INVALID_ARG
    # plain: too little workspace
    assert L.pkv_paged_attention_decode_prefix(*common, 0, 512, FAKE, 16, None, None) == \
        pkv.ERR_WORKSPACE


def test_empty_batch_is_a_no_op():
    assert decode(B=0, out=None, q=None) == pkv.OK


def test_workspace_size():
    # (B * Hq * parts) rows of (d + 2) floats, parts = ceil(W / (partition / 16))
    assert pkv.decode_workspace_bytes(8, 32, 128, 2048, 512) == 8 * 32 * 64 * 130 * 4
    assert pkv.decode_workspace_bytes(3, 4, 64, 33, 512) == 3 * 4 * 2 * 66 * 4
    assert pkv.decode_workspace_bytes(3, 4, 64, 33, 24) == 0  # not a multiple of 16
    assert pkv.decode_workspace_bytes(3, 0, 64, 33, 512) == 0


@pytest.mark.parametrize("args,code", [
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 100, 64), pkv.ERR_INVALID_ARG),   # head_dim % 8
    ((FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 128, 64), pkv.ERR_INVALID_ARG),
    ((None, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 64), pkv.ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE + 4, FAKE, FAKE, 4, 2, 128, 64), pkv.ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 0), pkv.ERR_INVALID_ARG),
    ((None, None, None, None, None, 0, 2, 128, 64), pkv.OK),                # nothing to write
])
def test_write_argument_checks(args, code):
    assert pkv.lib().pkv_paged_kv_write(*args, None, None) == code


def test_variant_choice_and_workspace_sizes():
    B, hq, hkv, d, W = 64, 32, 32, 128, 128
    split = pkv.decode_workspace_bytes_for(pkv.DECODE_SPLIT, B, hq, hkv, d, W)
    assert split == pkv.decode_workspace_bytes(B, hq, d, W)
    assert pkv.decode_workspace_bytes_for(pkv.DECODE_AUTO, B, hq, hkv, d, W) == max(split, 256)
    assert pkv.decode_workspace_bytes_for(pkv.DECODE_SINGLE, B, hq, hkv, d, W) == 256  # the order
    assert pkv.decode_workspace_bytes_for(pkv.DECODE_CLUSTER, B, hq, hkv, d, W) == 256
    assert pkv.decode_workspace_bytes_for(pkv.DECODE_CLUSTER, B, 28, 5, d, W) == 0  # 28 % 5
    assert pkv.decode_workspace_bytes_for(3, B, hq, hkv, d, W) == 0  # 3 is not a variant
    # enough units to fill the GPU: single pass, with or without workspace
    assert pkv.decode_variant_for(B, hq, hkv, d, W, 512, 0) == pkv.DECODE_SINGLE
    assert pkv.decode_variant_for(B, hq, hkv, d, W, 512, 1 << 40) == pkv.DECODE_SINGLE
    # long context (8 sequences x 2048 blocks, 8 x 8 units): a cluster part would span
    # 342 blocks, so split-K when the workspace holds its partials; the cluster
    # variant (6 parts: 64 x 6 CTAs in one wave of 3 per SM) without it
    long_split = pkv.decode_workspace_bytes(8, 32, d, 2048)
    assert pkv.decode_variant_for(8, 32, 8, d, 2048, 512, long_split) == pkv.DECODE_SPLIT
    assert pkv.decode_variant_for(8, 32, 8, d, 2048, 512, long_split - 1) == pkv.DECODE_CLUSTER
    assert pkv.decode_cluster_parts_for(8, 32, 8, d, 2048, pkv.DECODE_AUTO, 512, 0) == 6
    # one short sequence: the cluster variant, as many parts as one wave holds (<= 8)
    assert pkv.decode_variant_for(1, 32, 32, d, 128, 512, 0) == pkv.DECODE_CLUSTER
    assert pkv.decode_cluster_parts_for(1, 32, 32, d, 128, pkv.DECODE_AUTO, 512, 0) == 8
    assert pkv.decode_cluster_parts_for(4, 32, 32, d, 128, pkv.DECODE_AUTO, 512, 0) == 3
    # 8 sequences (256 units) leave no room for two parts each in one wave: split-K
    assert pkv.decode_cluster_parts_for(8, 32, 32, d, 128, pkv.DECODE_AUTO, 512, 0) == 0
    assert pkv.decode_variant_for(8, 32, 32, d, 128, 512, 1 << 30) == pkv.DECODE_SPLIT
    # ... never more parts than a quarter of the longest table's blocks
    assert pkv.decode_cluster_parts_for(1, 32, 32, d, 12, pkv.DECODE_AUTO, 512, 0) == 3
    assert pkv.decode_variant_for(1, 32, 32, d, 4, 512, 1 << 30) == pkv.DECODE_SINGLE
    # explicit cluster variant: the longest table cut into partition_tokens pieces, at most 8
    assert pkv.decode_cluster_parts_for(B, hq, hkv, d, W, pkv.DECODE_CLUSTER, 512, 0) == 4
    assert pkv.decode_cluster_parts_for(B, hq, hkv, d, W, pkv.DECODE_CLUSTER, 64, 0) == 8
    assert pkv.decode_cluster_parts_for(B, hq, hkv, d, 5, pkv.DECODE_CLUSTER, 512, 0) == 1
    assert pkv.decode_cluster_parts_for(B, hq, hkv, d, W, pkv.DECODE_SPLIT, 512, 0) == 0
    assert pkv.decode_variant_for(B, 5, 2, d, W, 512, 0) == -1
    assert decode(variant=3) == pkv.ERR_INVALID_ARG
    assert decode(variant=pkv.DECODE_SPLIT) == pkv.ERR_WORKSPACE
