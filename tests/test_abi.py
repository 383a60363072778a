"""The C-ABI library builds for sm_100a, loads, and exports every symbol its header declares.

No compute call runs here (there is no GPU): only host-side entry points and argument
checks that return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_rope_tile.h")


@pytest.fixture(scope="module")
def lib():
    from alibi_rope_tile_b200 import build
    path = build.build()
    import alibi_rope_tile_b200 as art
    assert os.path.samefile(path, art.LIB_PATH)
    return art.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("attn_prefill", "attn_decode", "attn_block", "attn_kv_append",
                 "attn_prefill_chunk", "attn_kv_write", "attn_decode_paged", "attn_kv_write_paged",
                 "attn_decode_latent", "attn_block_fused",
                 "attn_decode_workspace_size", "attn_block_workspace_size", "attn_alibi_slopes",
                 "attn_prefill_ws", "attn_prefill_workspace_size", "attn_prefill_host",
                 "attn_prefill_host_workspace_size",
                 "attn_sync_status", "attn_last_error", "attn_version"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    import alibi_rope_tile_b200 as art
    names = declared_functions()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"
    assert sorted(art.SIGNATURES) == names, "binding and header disagree on the entry points"


def test_library_is_sm100a_only():
    from alibi_rope_tile_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_alibi_slopes_host(lib, golden_dir):
    import alibi_rope_tile_b200 as art
    with open(os.path.join(golden_dir, "alibi_slopes.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for H, h, val in rows:
        assert art.alibi_slopes(int(H))[int(h)] == pytest.approx(float(val), rel=1e-7)


def test_version(lib):
    import alibi_rope_tile_b200 as art
    assert "sm_100a" in art.attn_version()


def test_workspace_sizes(lib):
    import alibi_rope_tile_b200 as art
    assert art.attn_decode_workspace_size(64, 32, 8, 128, 8192) > 0
    assert art.attn_decode_workspace_size(1, 3, 2, 8, 16) == 0          # H % KV != 0
    n = art.attn_block_workspace_size(1, 6, 32, 4, 2, 8, art.ATTN_F32)
    assert n >= 4 * (6 * 32 + 6 * 16 + 6 * 16 + 6 * 32)
    assert art.attn_block_workspace_size(1, 6, 32, 4, 2, 8, 7) == 0      # bad dtype


def _call_prefill(lib, **kw):
    a = dict(q=0x1000, k=0x1000, v=0x1000, out=0x1000, lse=None, B=1, T=8, H=4, KV=2, hd=8,
             pos0=0, base=10000.0, causal=1, window=0, slopes=None, dtype=1, stream=None)
    a.update(kw)
    return lib.attn_prefill(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["T"], a["H"],
                            a["KV"], a["hd"], a["pos0"], a["base"], a["causal"], a["window"],
                            a["slopes"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(H=6, KV=4), -1),             # H not a multiple of KV
    (dict(hd=7), -1),                  # odd head dimension
    (dict(hd=512), -1),                # beyond the maximum head dimension
    (dict(q=None), -1),                # NULL pointer
    (dict(k=0x1008), -2),              # not 16-byte aligned
    (dict(T=0), -1),                   # empty sequence
    (dict(causal=0, window=4), -1),    # window without the causal mask
    (dict(pos0=(1 << 24)), -1),        # positions beyond 2^24
    (dict(dtype=5), -1),               # unknown dtype
])
def test_prefill_argument_errors(lib, kw, code):
    import alibi_rope_tile_b200 as art
    assert _call_prefill(lib, **kw) == code
    buf = ctypes.create_string_buffer(256)
    assert lib.attn_last_error(buf, 256) == code
    assert len(buf.value) > 0
    with pytest.raises(art.AttnError):
        art._check(code)


def test_decode_workspace_error(lib):
    n = lib.attn_decode_workspace_size(2, 4, 2, 64, 128)
    st = lib.attn_decode(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, 2, 4, 2, 64, 128,
                         10000.0, 0, None, 1, 0x1000, n - 1, None)
    assert st == -6
    st = lib.attn_decode(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, 2, 4, 2, 48, 128,
                         10000.0, 0, None, 1, 0x1000, 1 << 30, None)
    assert st == -3      # hd = 48 is not a decode head size


def test_prefill_workspace_size_and_errors(lib):
    import alibi_rope_tile_b200 as art
    # the key rotation pass applies to bf16, hd 64 or 128, RoPE on: one turned copy of k
    assert lib.attn_prefill_workspace_size(2, 4096, 8, 128, 5e5, 1) == 2 * 4096 * 8 * 128 * 2
    assert lib.attn_prefill_workspace_size(2, 100, 3, 128, 1e4, 1) == 2 * 100 * 3 * 128 * 2
    assert lib.attn_prefill_workspace_size(2, 4096, 8, 128, 0.0, 1) == 0    # no rotation
    assert lib.attn_prefill_workspace_size(4, 1024, 16, 64, 1e4, 1) == 4 * 1024 * 16 * 64 * 2
    assert lib.attn_prefill_workspace_size(1, 64, 2, 32, 1e4, 1) == 0       # hd 32: in the kernel
    assert lib.attn_prefill_workspace_size(2, 64, 8, 128, 1e4, 0) == 0      # fp32
    assert lib.attn_prefill_workspace_size(0, 64, 8, 128, 1e4, 1) == 0      # invalid size
    assert art.attn_prefill_workspace_size(1, 10, 2, 128, 1e4) == 10 * 2 * 128 * 2
    need = lib.attn_prefill_workspace_size(1, 8, 2, 128, 1e4, 1)

    def call(ws, n, **kw):
        a = dict(B=1, T=8, H=4, KV=2, hd=128, base=1e4, window=0)
        a.update(kw)
        return lib.attn_prefill_ws(0x1000, 0x1000, 0x1000, 0x1000, None, a["B"], a["T"], a["H"],
                                   a["KV"], a["hd"], 0, a["base"], 1, a["window"], None, 1, ws, n, None)
    assert call(0x1000, need - 1) == -6          # workspace smaller than the size query
    assert call(0x1008, need) == -2              # misaligned workspace
    assert call(0x1000, need, H=6, KV=4) == -1   # argument errors come first
    assert call(0x1000, need, T=0) == -1


def test_prefill_host_workspace_and_errors(lib):
    import alibi_rope_tile_b200 as art
    n = lib.attn_prefill_host_workspace_size(2, 4096, 32, 8, 128, 5e5, 1)
    # dense device copies of q, k, v, out and lse, plus one slice's rotation scratch
    assert n >= 2 * 4096 * (2 * 32 + 2 * 8) * 128 * 2 + 2 * 32 * 4096 * 4
    assert lib.attn_prefill_host_workspace_size(2, 4096, 30, 8, 128, 5e5, 1) == 0   # H % KV
    assert lib.attn_prefill_host_workspace_size(0, 4096, 32, 8, 128, 5e5, 1) == 0   # B
    assert art.attn_prefill_host_workspace_size(5, 100, 8, 2, 64, 1e4) > 0
    need = lib.attn_prefill_host_workspace_size(1, 8, 4, 2, 128, 1e4, 1)

    def call(ws, nbytes, **kw):
        a = dict(B=1, T=8, H=4, KV=2, hd=128)
        a.update(kw)
        return lib.attn_prefill_host(0x1000, 0x1000, 0x1000, 0x1000, None, a["B"], a["T"], a["H"], a["KV"],
                                     a["hd"], 0, 1e4, 1, 0, None, 1, ws, nbytes, None)
    assert call(None, 0) == -6              # no workspace
    assert call(0x1000, need - 1) == -6     # too small
    assert call(0x1010, need) == -2         # not 256-byte aligned
    assert call(0x1000, need, H=6, KV=4) == -1
    assert call(0x1000, need, hd=7) == -1


def test_block_workspace_error(lib):
    st = lib.attn_block(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 1, 6, 32, 4, 2, 8, 0,
                        10000.0, 1, 0, None, 0, 0x1000, 16, None)
    assert st == -6


def test_chunk_and_kv_write_argument_errors(lib):
    P = 0x1000
    def chunk(**kw):
        a = dict(seqlens=P, qpos0=P, B=2, Tq=16, H=8, KV=2, hd=128, Lmax=64, causal=1, window=0,
                 dtype=1)
        a.update(kw)
        return lib.attn_prefill_chunk(P, P, P, a["seqlens"], a["qpos0"], P, None, a["B"], a["Tq"],
                                      a["H"], a["KV"], a["hd"], a["Lmax"], 10000.0, a["causal"],
                                      a["window"], None, a["dtype"], None)
    assert chunk(seqlens=None) == -1                 # NULL lengths
    assert chunk(causal=0, window=8) == -1          # a window needs the causal mask
    assert chunk(Lmax=0) == -1
    assert chunk(H=6, KV=4) == -1                   # H % KV
    assert chunk(dtype=0) == -3                     # fp32 has no chunk kernel
    assert chunk(hd=48) == -3                       # neither has hd 48
    def write(**kw):
        a = dict(B=2, Tn=4, KV=2, hd=64, Lmax=64)
        a.update(kw)
        return lib.attn_kv_write(P, P, P, P, P, a["B"], a["Tn"], a["KV"], a["hd"], a["Lmax"],
                                 10000.0, 1, None)
    assert write(Tn=0) == -1
    assert write(Tn=70000) == -1
    assert write(hd=7) == -1


def test_paged_argument_errors(lib):
    P = 0x1000
    def dec(**kw):
        a = dict(B=2, H=8, KV=2, hd=128, ps=16, npages=64, mb=8, dtype=1, table=P)
        a.update(kw)
        return lib.attn_decode_paged(P, P, P, a["table"], P, P, P, None, a["B"], a["H"], a["KV"], a["hd"],
                                     a["ps"], a["npages"], a["mb"], 10000.0, 0, None, a["dtype"], P,
                                     1 << 30, None)
    assert dec(ps=24) == -1          # page size not a power of two dividing 128
    assert dec(ps=256) == -1
    assert dec(npages=0) == -1
    assert dec(table=None) == -1
    assert dec(dtype=0) == -3        # fp32 has no paged kernel
    assert dec(hd=32) == -3
    def write(**kw):
        a = dict(Tn=4, ps=64)
        a.update(kw)
        return lib.attn_kv_write_paged(P, P, P, P, P, P, 2, a["Tn"], 2, 64, a["ps"], 8, 4, 10000.0, 1,
                                       None)
    assert write(Tn=0) == -1
    assert write(ps=4) == -1


def test_latent_argument_errors(lib):
    P = 0x1000
    def lat(**kw):
        a = dict(H=32, hd=128, dc=128, dtype=1, W=P)
        a.update(kw)
        return lib.attn_decode_latent(P, P, a["W"], P, P, P, P, None, 4, a["H"], a["hd"], a["dc"], 256, 0,
                                      None, a["dtype"], P, 1 << 30, None)
    assert lat(W=None) == -1
    assert lat(dc=96) == -3          # the latent decode runs dc 64 or 128
    assert lat(H=64) == -3           # one key/value head serves at most 32 query heads here
    assert lat(dtype=0) == -3
    assert lib.attn_decode_latent_workspace_size(4, 32, 128, 96, 256) == 0
    assert lib.attn_decode_latent_workspace_size(4, 32, 128, 64, 256) > 0


def test_fused_block_argument_errors(lib):
    P = 0x1000
    def fused(**kw):
        a = dict(gamma=P, kc=None, vc=None, Lmax=0, T=16, d=512, H=8, KV=2, hd=64, pos0=0, dtype=1)
        a.update(kw)
        return lib.attn_block_fused(P, a["gamma"], P, P, P, a["kc"], a["vc"], a["Lmax"], 2, a["T"], a["d"],
                                    a["H"], a["KV"], a["hd"], a["pos0"], 10000.0, 1, 0, None, 1e-6,
                                    a["dtype"], P, 1 << 30, None)
    assert fused(kc=P) == -1                          # one cache without the other
    assert fused(kc=P, vc=P, Lmax=20, pos0=8) == -1   # slots pos0..pos0+T-1 exceed the cache
    assert fused(d=500) == -1                         # d not a multiple of 8
    assert fused(hd=32, d=256) == -3                  # head size without a tensor-core path
    assert fused(dtype=0) == -3
    assert lib.attn_block_fused_workspace_size(2, 16, 512, 8, 2, 64) > 0
    # gamma = NULL means "already folded into Wqkv"; the folding entry point checks its own
    assert lib.attn_fold_rmsnorm_gamma(None, P, P, 512, 768, None) == -1
    assert lib.attn_fold_rmsnorm_gamma(P, P, P, 512, 770, None) == -1   # N not a multiple of 8
    assert lib.attn_fold_rmsnorm_gamma(P + 4, P, P, 512, 768, None) == -2  # misaligned


def test_binding_requires_cuda_tensors(lib):
    import torch
    import alibi_rope_tile_b200 as art
    q = torch.zeros(1, 4, 2, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        art.attn_prefill(q, q, q, out=q)


def test_binding_rejects_mismatched_shapes(lib):
    """The binding checks every tensor's shape against the sizes it passes to the library
    before any call: the kernels index by those sizes, so a tensor of another shape would be
    read or written out of bounds. (CPU tensors: the shape check fires before the device check.)"""
    import torch

    import alibi_rope_tile_b200 as art
    bf = torch.bfloat16
    B, T, d, H, KV, hd = 2, 16, 64, 4, 2, 16
    x = torch.zeros(B, T, d, dtype=bf)
    gamma = torch.ones(d, dtype=bf)
    Wqkv = torch.zeros(d, (H + 2 * KV) * hd, dtype=bf)
    Wo = torch.zeros(H * hd, d, dtype=bf)
    kc = torch.zeros(B, 32, KV, hd, dtype=bf)
    cases = [
        (dict(Wqkv=torch.zeros(d, (H + 2 * KV) * hd + 1, dtype=bf)), "Wqkv"),
        (dict(Wqkv=torch.zeros(d + 8, (H + 2 * KV) * hd, dtype=bf)), "Wqkv"),
        (dict(Wo=torch.zeros(H * hd, d + 8, dtype=bf)), "Wo"),
        (dict(gamma=torch.ones(d - 8, dtype=bf)), "gamma"),
        (dict(kcache=torch.zeros(B, 32, KV + 1, hd, dtype=bf), vcache=kc), "kcache"),
        (dict(kcache=kc, vcache=torch.zeros(B, 31, KV, hd, dtype=bf)), "vcache"),
        (dict(kcache=kc, vcache=None), "both"),
    ]
    for change, what in cases:
        kw = dict(x=x, gamma=gamma, Wqkv=Wqkv, Wo=Wo, kcache=None, vcache=None)
        kw.update(change)
        with pytest.raises(ValueError, match=what):
            art.attn_block_fused(kw.pop("x"), kw.pop("gamma"), kw.pop("Wqkv"), kw.pop("Wo"), H=H, KV=KV, **kw)
    Wq, Wk = torch.zeros(d, H * hd, dtype=bf), torch.zeros(d, KV * hd, dtype=bf)
    with pytest.raises(ValueError, match="Wv"):
        art.attn_block(x, Wq, Wk, torch.zeros(d, KV * hd + 8, dtype=bf), Wo, H=H, KV=KV)
    with pytest.raises(ValueError, match="Wo"):
        art.attn_block(x, Wq, Wk, Wk, torch.zeros(H * hd + 8, d, dtype=bf), H=H, KV=KV)
    q = torch.zeros(B, T, H, hd, dtype=bf)
    k = torch.zeros(B, T, KV, hd, dtype=bf)
    with pytest.raises(ValueError, match="out"):
        art.attn_prefill(q, k, k, out=torch.zeros(B, T, H, hd + 8, dtype=bf))
    with pytest.raises(ValueError, match="lse"):
        art.attn_prefill(q, k, k, lse=torch.zeros(B, T, H, dtype=torch.float32))
    dq = torch.zeros(B, H, hd, dtype=bf)
    sl = torch.zeros(B, dtype=torch.int32)
    with pytest.raises(ValueError, match="vcache"):
        art.attn_decode(dq, kc, torch.zeros(B, 16, KV, hd, dtype=bf), sl, sl)
    with pytest.raises(ValueError, match="seqlens"):
        art.attn_decode(dq, kc, kc, torch.zeros(B + 1, dtype=torch.int32), sl)
    with pytest.raises(ValueError, match="out"):
        art.attn_decode_noalloc(dq, kc, kc, sl, sl, None)
    with pytest.raises(ValueError, match="qpos0"):
        art.attn_prefill_chunk(q, kc, kc, sl, torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="kcache"):
        art.attn_kv_write(k, k, torch.zeros(B, 32, KV, hd + 2, dtype=bf), kc, sl)
    with pytest.raises(ValueError, match="block_table"):
        art.attn_decode_paged(dq, kc, kc, torch.zeros(B + 1, 4, dtype=torch.int32), sl, sl)
    with pytest.raises(ValueError, match="W_uv"):
        art.attn_decode_latent(dq, torch.zeros(B, 32, 64, dtype=bf), torch.zeros(H, 64, hd, dtype=bf),
                               torch.zeros(H, 64, hd + 2, dtype=bf), sl, sl)
    with pytest.raises(ValueError, match="pos"):
        art.attn_kv_append(dq[:, :KV], dq[:, :KV], kc, kc, torch.zeros(B + 1, dtype=torch.int32))


def _host_plan_bytes(B, T, H, KV, hd, rope_base, dtype):
    """The host-buffer prefill's device scratch, restated: the slices (runs of at most eight
    groups of whole sequences when B >= 4; else one sequence and the largest key/value-head
    group giving 4 to 16 slices), the last slice cut into a slice per sequence and halving head
    groups; per slice dense q, k, v, out and lse (each rounded to 256 bytes), plus the rotation
    scratch of the largest slice (bf16, hd 64/128, RoPE only)."""
    r256 = lambda n: (n + 255) // 256 * 256
    es = 4 if dtype == 0 else 2
    G = H // KV
    sl = []
    if B >= 4:
        runs = min(B, 8)
        nbs = (B + runs - 1) // runs
        sl = [(b0, min(nbs, B - b0), 0, KV) for b0 in range(0, B, nbs)]
    else:
        ng = KV
        for g in range(KV, 0, -1):
            if KV % g == 0 and B * (KV // g) >= 4:
                if B * (KV // g) <= 16:
                    ng = g
                break
        sl = [(b, 1, g0, ng) for b in range(B) for g0 in range(0, KV, ng)]
    b0, nb, g0, ng = sl.pop()
    if nb > 1:
        sl.append((b0, nb - 1, 0, KV))
        b0, nb, g0, ng = b0 + nb - 1, 1, 0, KV
    rem = ng
    while rem > 1:
        part = (rem + 1) // 2
        sl.append((b0, 1, g0, part))
        g0 += part
        rem -= part
    if rem == 1:
        sl.append((b0, 1, g0, 1))
    total = 0
    rot = 0
    for (_, nb, _, ng) in sl:
        q = r256(nb * T * ng * G * hd * es)
        kv = r256(nb * T * ng * hd * es)
        lse = r256(nb * ng * G * T * 4)
        total += 2 * q + 2 * kv + lse
        if dtype == 1 and hd in (64, 128) and rope_base > 0:
            rot = max(rot, nb * T * ng * hd * 2)
    return total + r256(rot), len(sl)


@pytest.mark.parametrize("shape", [(2, 4096, 32, 8, 128, 5e5, 1), (1, 257, 8, 2, 128, 5e5, 1),
                                   (3, 130, 8, 1, 128, 1e4, 1), (5, 200, 4, 2, 64, 0.0, 1),
                                   (18, 40, 4, 4, 128, 1e4, 0), (1, 90, 12, 4, 64, 1e4, 0),
                                   (2, 300, 16, 8, 128, 1e4, 1), (1, 64, 7, 7, 64, 1e4, 1)])
def test_prefill_host_workspace_follows_the_slice_plan(lib, shape):
    B, T, H, KV, hd, base, dtype = shape
    want, nslices = _host_plan_bytes(B, T, H, KV, hd, base, dtype)
    assert nslices <= 32
    assert lib.attn_prefill_host_workspace_size(B, T, H, KV, hd, base, dtype) == want
