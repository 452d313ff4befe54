"""Host-side checks of libmoe that need no GPU: the library loads, exports every symbol
include/moe.h declares, computes the same capacities as the oracle, and rejects bad
arguments with status codes (never by crashing)."""
import ctypes
import os
import re

import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    from capacity_limited_routed_b200 import moe
    return moe


def test_header_and_binding_agree_on_exports(M):
    with open(os.path.join(ROOT, "include", "moe.h"), encoding="utf-8") as f:
        hdr = f.read()
    declared = set(re.findall(r"^MOE_API\s+(?:moe_status_t|const char\*|int64_t)\s+(moe_\w+)\s*\(", hdr, re.M))
    assert declared == set(M.EXPORTS)
    lib = ctypes.CDLL(M.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_plan_capacities_match_oracle(M, wid):
    s = synth.WORKLOADS[wid]
    plan = M.Plan.from_shape(s)
    g = O.geometry(s)
    assert (plan.info.cap_send, plan.info.cap_recv) == (g.C_s, g.C_r)
    assert plan.info.local_experts == g.L and plan.info.experts_per_wave == g.P
    assert plan.info.n_pools == g.D * g.W
    assert plan.info.pool_row_elems == s.d_latent + 8
    assert plan.info.pools_bytes == g.D * g.W * g.C_s * (s.d_latent + 8) * 2
    assert plan.info.expert_out_bytes == s.n_experts * g.C_r * s.d_latent * 2
    assert plan.info.stats_bytes == 4 * (8 + 4 * s.n_experts + g.D * g.W)
    assert plan.info.workspace_bytes % 256 == 0 and plan.info.saved_bytes % 256 == 0


def test_plan_rejects_bad_shapes(M):
    base = dict(T=64, d_model=128, d_latent=64, n_experts=24, top_k=2, n_dest=4, hidden_routed=128,
                n_shared=1, hidden_shared=128)
    M.Plan(**base)
    bad = [
        (dict(n_experts=25), M.STATUS[2]),            # E % D
        (dict(n_dest=8), M.STATUS[2]),                # E/D = 3 = W but (E/D) % W ok? 24/8 = 3 -> P = 1: valid
        (dict(d_model=100), M.STATUS[2]),
        (dict(hidden_routed=64), M.STATUS[2]),
        (dict(top_k=0), M.STATUS[1]),
        (dict(top_k=33, n_experts=48, n_dest=4), M.STATUS[2]),
        (dict(T=-1), M.STATUS[1]),
    ]
    for kw, _ in bad:
        args = dict(base, **kw)
        if kw == dict(n_dest=8):
            M.Plan(**args)                            # 24 experts over 8 destinations of 3 waves is fine
            continue
        with pytest.raises(M.MoEError):
            M.Plan(**args)
    with pytest.raises(M.MoEError) as ei:
        M.Plan(**dict(base, cap_send=(0, 100)))
    assert ei.value.code == 1


def test_empty_batch_plan(M):
    p = M.Plan(T=0, d_model=128, d_latent=64, n_experts=24, top_k=2, n_dest=4, hidden_routed=128,
               n_shared=1, hidden_shared=128)
    assert p.info.cap_send >= 1 and p.info.cap_recv >= 1


def test_compute_calls_fail_cleanly_without_a_device(M):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = M.Plan.from_shape(synth.TINY)
    lib = M.lib()
    fake = ctypes.c_void_p(0x1000)
    code = lib.moe_route(p.handle, fake, fake, fake, fake, fake, None)
    assert code == 2 and "device" in M.moe_last_error()
    code = lib.moe_bias_update(p.handle, fake, fake, ctypes.c_float(1e-3), None)
    assert code == 2
    code = lib.moe_gemm_bf16(128, 128, 64, fake, 0, fake, 0, fake, 1, None, None)
    assert code == 2


def test_null_arguments_are_rejected(M):
    p = M.Plan.from_shape(synth.TINY)
    lib = M.lib()
    assert lib.moe_route(p.handle, None, None, None, None, None, None) == 1
    assert lib.moe_forward(p.handle, None, None, None, None, None, None, None, None, 0, None) == 1
    w = M.moe_weights_t()
    assert lib.moe_forward(p.handle, ctypes.byref(w), None, None, None, None, None, None, None, 0, None) == 1
    assert lib.moe_gemm_bf16(0, 8, 8, None, 0, None, 0, None, 1, None, None) == 1
    fake = ctypes.c_void_p(0x1000)
    # too-small workspace is reported before anything runs
    assert lib.moe_dispatch(p.handle, fake, fake, fake, fake, fake, fake, 16, None) == 3


def test_side_stream_switch_rejects_other_values(M):
    lib = M.lib()
    assert lib.moe_set_side_stream(2) == 1 and lib.moe_set_side_stream(-1) == 1
    assert lib.moe_set_side_stream(0) == 0 and lib.moe_set_side_stream(1) == 0


def test_dropless_plan_sizes(M):
    """Both capacity numerators 0 select the dropless variant: no caps, pools packed to
    T*k rows, expert buffers packed by expert with each expert padded to 128 rows."""
    T, k, E, dl = 300, 3, 24, 64
    p = M.Plan(T=T, d_model=128, d_latent=dl, n_experts=E, top_k=k, n_dest=4, hidden_routed=128,
               n_shared=1, hidden_shared=128, cap_send=(0, 1), cap_recv=(0, 1))
    assert p.info.cap_send == 0 and p.info.cap_recv == 0
    assert p.info.pools_bytes == T * k * (dl + 8) * 2
    assert p.info.expert_out_bytes == (T * k + 127 * E) * dl * 2
    # only one numerator 0 is an error, as before
    with pytest.raises(M.MoEError):
        M.Plan(T=T, d_model=128, d_latent=dl, n_experts=E, top_k=k, n_dest=4, hidden_routed=128,
               n_shared=1, hidden_shared=128, cap_send=(0, 1))


def test_plan_with_sources(M):
    """S sources: per-source sender caps, S*D*W pools; T/S must be whole scan chunks."""
    base = dict(T=512, d_model=128, d_latent=64, n_experts=24, top_k=2, n_dest=4, hidden_routed=128,
                n_shared=1, hidden_shared=128)
    for S in (1, 2, 4, 16):
        p = M.Plan(**base, n_sources=S)
        assert p.info.n_pools == S * 4 * 3
        assert p.info.cap_send == -(-512 * 2 * 110 // (100 * 12 * S))
        assert p.info.cap_recv == -(-512 * 2 * 115 // (100 * 24))
        assert p.info.pools_bytes == S * 12 * p.info.cap_send * (64 + 8) * 2
    with pytest.raises(M.MoEError):
        M.Plan(**base, n_sources=3)    # 512 / 3 is not whole
    with pytest.raises(M.MoEError):
        M.Plan(**base, n_sources=32)   # 16 tokens per source: not whole 32-token chunks


def test_struct_layouts_match_the_header(M, tmp_path):
    """Every struct the binding passes across the ABI has the size and field offsets the
    header gives it, as compiled by the host C compiler."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = [M.moe_config_t, M.moe_plan_info_t, M.moe_weights_t, M.moe_grads_t, M.moe_expert_weights_t,
               M.moe_profile_record_t, M.moe_saved_view_t]
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{os.path.join(ROOT, "include", "moe.h")}"',
             "int main(void) {"]
    for st in structs:
        n = st.__name__
        lines.append(f'  printf("{n} size %zu\\n", sizeof({n}));')
        for f, _ in st._fields_:
            lines.append(f'  printf("{n} {f} %zu\\n", offsetof({n}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c11", "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {" ".join(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for st in structs:
        n = st.__name__
        assert got[f"{n} size"] == ctypes.sizeof(st), n
        for f, _ in st._fields_:
            assert got[f"{n} {f}"] == getattr(st, f).offset, (n, f)
