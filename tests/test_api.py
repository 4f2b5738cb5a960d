"""The C ABI without a GPU: the library loads, exports what include/ba.h
declares, sizes workspaces, and rejects bad arguments on the host before it
would launch anything."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_kunlun_b200 as ba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ba_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ba.library_path())
    names = declared_functions()
    assert {"ba_fwd", "ba_bwd", "ba_fwd_workspace_size", "ba_bwd_workspace_size",
            "ba_device_status", "ba_status_string", "ba_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libba.so does not export {n}"


def test_status_strings_and_version():
    assert ba.ba_status_string(ba.BA_OK) == "ok"
    assert "timed out" in ba.ba_status_string(ba.BA_ERR_TIMEOUT)
    assert ba.ba_status_string(99) == "unknown status"
    assert ba.ba_version() >= 100


def prob(batch=2, T=300, H=4, D=64, dt=ba.BA_BF16):
    return ba.BAProblem(batch, T, H, D, dt)


def test_workspace_sizes():
    p = prob(batch=3, T=1000, H=2, D=128)
    f = ba.ba_fwd_workspace_size(p, 128, 2)
    b = ba.ba_bwd_workspace_size(p, 128, 2)
    assert f >= 256 + 4 * 4 and f % 256 == 0
    # backward adds two per-row float buffers (Delta and lse for the dK/dV pass), H*T floats each,
    # and (bf16) 128 staged rows of q and of dout per example
    staged = 2 * 3 * 128 * 2 * 128 * 2
    assert f + 2 * 4 * 2 * 1000 + staged <= b <= f + 2 * 4 * 2 * 1000 + staged + 1024
    # window 1 with blocks dividing 128 (each query tile sees only its own key tile): the fused
    # backward stages the partial key tiles (k) as well; other masks do not
    for blk in (1, 16, 64, 128):
        assert ba.ba_bwd_workspace_size(p, blk, 1) == b + staged // 2
        assert ba.ba_mx_bwd_workspace_size(p, blk, 1) == ba.ba_mx_bwd_workspace_size(p, 128, 2) + staged // 2
    for blk, win in ((96, 1), (256, 1), (64, 2)):
        assert ba.ba_bwd_workspace_size(p, blk, win) == b
    # float32 has no staged rows
    p32 = prob(batch=3, T=1000, H=2, D=64, dt=ba.BA_F32)
    f32, b32 = ba.ba_fwd_workspace_size(p32, 128, 2), ba.ba_bwd_workspace_size(p32, 128, 2)
    assert f32 + 2 * 4 * 2 * 1000 <= b32 <= f32 + 2 * 4 * 2 * 1000 + 512
    assert ba.ba_bwd_workspace_size(p32, 64, 1) == b32
    # the generalized attention's workspace (either direction) is the backward's
    assert ba.ba_gdpa_workspace_size(p, 128, 2) == f + staged
    # the work table grows with the number of 128-row tiles
    assert ba.ba_fwd_workspace_size(prob(batch=3, T=100000, H=2, D=128), 128, 2) >= 16 * (100000 // 128)
    assert ba.ba_fwd_workspace_size(prob(batch=-1), 128, 2) == 0
    assert ba.ba_fwd_workspace_size(p, 0, 2) == 0
    assert ba.ba_fwd_workspace_size(p, 128, 0) == 0


FAKE = 1 << 20  # a 256-byte-aligned address that is never dereferenced on invalid arguments


def call_fwd(p, block=128, window=2, q=FAKE, k=FAKE, v=FAKE, offs=FAKE, out=FAKE, lse=FAKE,
             ws=FAKE, ws_bytes=1 << 30):
    lib = ba._load()
    return lib.ba_fwd(ctypes.byref(p) if p is not None else None, q, k, v, offs, block, window, None,
                      out, lse, ws, ws_bytes, None)


def call_bwd(p, block=128, window=2, ptrs=None, ws=FAKE, ws_bytes=1 << 30):
    lib = ba._load()
    d = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, offs=FAKE, dq=FAKE, dk=FAKE, dv=FAKE)
    d.update(ptrs or {})
    return lib.ba_bwd(ctypes.byref(p), d["q"], d["k"], d["v"], d["out"], d["lse"], d["dout"], d["offs"],
                      block, window, None, d["dq"], d["dk"], d["dv"], ws, ws_bytes, None)


@pytest.mark.parametrize("kw", [
    dict(p=None),
    dict(block=0), dict(window=0), dict(block=-5),
    dict(q=0), dict(k=0), dict(v=0), dict(out=0), dict(lse=0), dict(offs=0),
    dict(q=FAKE + 8), dict(out=FAKE + 4), dict(lse=FAKE + 2), dict(offs=FAKE + 2),
    dict(ws=0), dict(ws=FAKE + 128), dict(ws_bytes=16),
])
def test_fwd_rejects_invalid_arguments(kw):
    p = kw.pop("p", prob())
    assert call_fwd(p, **kw) == ba.BA_ERR_INVALID_ARG


@pytest.mark.parametrize("p", [prob(batch=-1), prob(T=-1), prob(H=0), prob(D=0), prob(batch=0, T=5),
                               ba.BAProblem(2, 300, 4, 64, 7)])
def test_fwd_rejects_invalid_problems(p):
    assert call_fwd(p) == ba.BA_ERR_INVALID_ARG


@pytest.mark.parametrize("p", [prob(D=32), prob(D=96), prob(D=256), prob(D=128, dt=ba.BA_F32),
                               prob(D=48, dt=ba.BA_F32)])
def test_unsupported_head_dims(p):
    assert call_fwd(p) == ba.BA_ERR_UNSUPPORTED
    assert call_bwd(p) == ba.BA_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["q", "k", "v", "out", "lse", "dout", "offs", "dq", "dk", "dv"])
def test_bwd_rejects_null_pointers(name):
    assert call_bwd(prob(), ptrs={name: 0}) == ba.BA_ERR_INVALID_ARG


def test_bwd_rejects_small_workspace():
    p = prob(batch=2, T=300, H=4, D=64)
    need = ba.ba_bwd_workspace_size(p, 128, 2)
    assert call_bwd(p, ws_bytes=need - 1) == ba.BA_ERR_INVALID_ARG


# ------------------------------------------------------------- rotary ---

def test_rope_workspace_sizes():
    p = prob(batch=3, T=1000, H=2, D=128)
    for plain, rope, esz in ((ba.ba_fwd_workspace_size, ba.ba_rope_fwd_workspace_size, 2),
                             (ba.ba_bwd_workspace_size, ba.ba_rope_bwd_workspace_size, 2)):
        extra = 2 * ((1000 * 2 * 128 * esz + 255) // 256 * 256)   # rotated copies of q and k
        assert rope(p, 128, 2) == plain(p, 128, 2) + extra
    p32 = prob(batch=1, T=77, H=3, D=32, dt=ba.BA_F32)
    assert ba.ba_rope_fwd_workspace_size(p32, 64, 1) == \
        ba.ba_fwd_workspace_size(p32, 64, 1) + 2 * ((77 * 3 * 32 * 4 + 255) // 256 * 256)
    assert ba.ba_rope_fwd_workspace_size(prob(batch=-1), 128, 2) == 0
    assert ba.ba_rope_bwd_workspace_size(p, 128, 0) == 0


def test_rope_rejects_bad_arguments_before_launching():
    p = prob(batch=2, T=300, H=4, D=64)
    need_f = ba.ba_rope_fwd_workspace_size(p, 128, 2)
    need_b = ba.ba_rope_bwd_workspace_size(p, 128, 2)
    good = ba.BARope(FAKE, FAKE, 300)

    def fwd(rope, ws_bytes=need_f):
        return ba.ba_rope_fwd(p, rope, FAKE, FAKE, FAKE, FAKE, 128, 2, None, FAKE, FAKE, FAKE,
                              workspace_bytes=ws_bytes, stream=0)

    def bwd(rope, ws_bytes=need_b):
        return ba.ba_rope_bwd(p, rope, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 2, None, FAKE, FAKE, FAKE,
                              FAKE, workspace_bytes=ws_bytes, stream=0)

    for call in (fwd, bwd):
        assert call(None) == ba.BA_ERR_INVALID_ARG                                   # no tables
        assert call(ba.BARope(None, FAKE, 300)) == ba.BA_ERR_INVALID_ARG             # null cos
        assert call(ba.BARope(FAKE, None, 300)) == ba.BA_ERR_INVALID_ARG             # null sin
        assert call(ba.BARope(FAKE + 8, FAKE, 300)) == ba.BA_ERR_INVALID_ARG         # misaligned
        assert call(ba.BARope(FAKE, FAKE, 0)) == ba.BA_ERR_INVALID_ARG               # no rows
    # the plain entry points' workspace is too small: the rotated copies need room
    assert fwd(good, ba.ba_fwd_workspace_size(p, 128, 2)) == ba.BA_ERR_INVALID_ARG
    assert bwd(good, need_b - 1) == ba.BA_ERR_INVALID_ARG


def test_rope_saved_copies_must_come_in_pairs():
    p = prob(batch=2, T=300, H=4, D=64)
    need_b = ba.ba_rope_bwd_workspace_size(p, 128, 2)
    for rope in (ba.BARope(FAKE, FAKE, 300, FAKE, None), ba.BARope(FAKE, FAKE, 300, None, FAKE),
                 ba.BARope(FAKE, FAKE, 300, FAKE + 4, FAKE), ba.BARope(FAKE, FAKE, 300, FAKE, FAKE + 2)):
        assert ba.ba_rope_fwd(p, rope, FAKE, FAKE, FAKE, FAKE, 128, 2, None, FAKE, FAKE, FAKE,
                              workspace_bytes=need_b, stream=0) == ba.BA_ERR_INVALID_ARG
        assert ba.ba_rope_bwd(p, rope, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 2, None, FAKE, FAKE, FAKE,
                              FAKE, workspace_bytes=need_b, stream=0) == ba.BA_ERR_INVALID_ARG


def test_header_is_c99_and_a_c_client_links(tmp_path):
    """tests/c/abi_check.c: a plain-C client compiled with -std=c99 -pedantic
    against include/ba.h and linked against libba.so; it runs only calls that
    never reach the device (sizes, status strings, argument errors)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(ba.library_path())
    exe = str(tmp_path / "abi_check")
    subprocess.run([cc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(root, "include"), os.path.join(root, "tests", "c", "abi_check.c"),
                    "-o", exe, "-L", lib_dir, "-l:libba.so", f"-Wl,-rpath,{lib_dir}"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "all checks passed" in r.stdout
