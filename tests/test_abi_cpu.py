"""The C-ABI library on the host: loads, exports every declared symbol, and its
host logic (validation, planning, status strings) behaves as the header says.
No kernel is launched here."""
import ctypes
import os
import subprocess

import pytest
import torch

import moe_router_gating_b200 as tk
from moe_router_gating_b200 import build as tkbuild


@pytest.fixture(scope="module", autouse=True)
def built():
    tkbuild.build()


def test_exports_every_declared_symbol():
    declared = tk.exported_symbols()
    assert "tk_gating_fused_topk" in declared and len(declared) >= 6
    lib = tk.library()
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", tk.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(declared) <= exported, set(declared) - exported
    # nothing else with C linkage leaks out under the library prefix
    assert {s for s in exported if s.startswith("tk_")} == set(declared)


def test_status_strings():
    for code in (tk.TK_OK, tk.TK_ERR_INVALID_ARG, tk.TK_ERR_UNSUPPORTED, tk.TK_ERR_ALIGNMENT, tk.TK_ERR_CUDA,
                 tk.TK_ERR_DEVICE_TIMEOUT):
        assert tk.status_string(code).startswith("TK_")
    assert tk.status_string(12345) == "unknown tk_status"


@pytest.mark.parametrize("args,code", [
    ((-1, 64, 16, 2), tk.TK_ERR_INVALID_ARG),       # negative T
    ((8, 0, 16, 2), tk.TK_ERR_INVALID_ARG),         # H < 1
    ((8, 64, 16, 0), tk.TK_ERR_INVALID_ARG),        # k < 1
    ((8, 64, 16, 17), tk.TK_ERR_INVALID_ARG),       # k > E
    ((8, 60, 16, 2), tk.TK_ERR_UNSUPPORTED),        # H % 8
    ((8, 64, 20, 2), tk.TK_ERR_UNSUPPORTED),        # E % 8
    ((8, 64, 8, 2), tk.TK_ERR_UNSUPPORTED),         # E < 16
    ((8, 64, 1032, 2), tk.TK_ERR_UNSUPPORTED),      # E > 1024
    ((8, 64, 64, 33), tk.TK_ERR_UNSUPPORTED),       # k > 32
])
def test_invalid_sizes_rejected_before_cuda(args, code):
    T, H, E, k = args
    assert tk.fused_topk_gating_ptr(16, 16, T, H, E, k, 16, 16) == code
    with pytest.raises(tk.TkGatingError) as ei:
        tk.make_plan(T, H, E, k)
    assert ei.value.status == code


def test_null_and_misaligned_pointers():
    assert tk.fused_topk_gating_ptr(0, 16, 8, 64, 16, 2, 16, 16) == tk.TK_ERR_INVALID_ARG
    assert tk.fused_topk_gating_ptr(16, 16, 8, 64, 16, 2, 0, 16) == tk.TK_ERR_INVALID_ARG
    assert tk.fused_topk_gating_ptr(18, 16, 8, 64, 16, 2, 16, 16) == tk.TK_ERR_ALIGNMENT
    assert tk.fused_topk_gating_ptr(16, 16, 8, 64, 16, 2, 16, 20) == tk.TK_ERR_ALIGNMENT


def test_zero_tokens_is_a_no_op():
    # T == 0: TK_OK without touching pointers or the device
    assert tk.fused_topk_gating_ptr(0, 0, 0, 64, 16, 2, 0, 0) == tk.TK_OK
    assert tk.make_plan(0, 64, 16, 2)["variant"] == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_no_cpu_fallback_without_gpu():
    assert tk.fused_topk_gating_ptr(16, 16, 8, 64, 16, 2, 16, 16) in (tk.TK_ERR_CUDA, tk.TK_ERR_UNSUPPORTED)


def test_plans_for_router_workloads():
    import workloads
    for wl in workloads.WORKLOADS.values():
        p = tk.make_plan(wl.T, wl.H, wl.E, wl.k, 148)
        assert p["variant"] in (1, 2, 3)
        assert p["n_pad"] % 16 == 0 and p["n_pad"] >= wl.E
        assert p["smem_bytes"] <= 232448
        assert p["tmem_cols"] in (32, 64, 128, 256, 512)
        assert p["grid"] >= 1 and p["grid"] % max(p["cluster"], 1) == 0
        assert p["stages"] >= 2
        if p["variant"] == 1:
            assert p["grid"] == min(p["num_tiles"], 148) and p["cluster"] == 1
        if p["variant"] == 3:
            assert p["cluster"] == 2 and p["block_m"] == 256 and p["n_pad"] % 128 == 0 and p["n_pad"] <= 1024
            assert p["grid"] == 2 * min(p["num_tiles"], 74)
        if p["variant"] == 2:
            C = p["cluster"]
            assert C in (2, 4, 8, 16) and p["split_h"] == C and C <= p["k_blocks"]
            assert p["grid"] == p["num_tiles"] * C <= 148


def test_plan_half_tiles_cover_rows_once():
    for T in (9473, 18945, 19999, 20000, 30000, 60000, 65536, 100000):
        p = tk.make_plan(T, 512, 256, 8, 148)
        if p["variant"] != 3:
            continue
        pairs = p["grid"] // 2
        rows = p["num_tiles"] * 256 + p["num_half_tiles"] * 128
        assert rows >= T and rows - T < 256
        assert p["num_half_tiles"] <= pairs
        if p["num_half_tiles"]:
            assert p["num_tiles"] % pairs == 0  # every pair: the same full tiles, then one half tile


def test_plan_variant_choice():
    # few tiles: split H across a cluster; many tiles: persistent row tiles / pairs
    assert tk.make_plan(1, 7168, 256, 8)["variant"] == 2
    assert tk.make_plan(1, 7168, 256, 8)["cluster"] == 16
    assert tk.make_plan(4096, 7168, 256, 8)["cluster"] == 4
    assert tk.make_plan(8192, 7168, 256, 8)["cluster"] == 2
    assert tk.make_plan(65536, 7168, 256, 8)["variant"] == 3
    assert tk.make_plan(16384, 4096, 64, 6)["variant"] == 1
    assert tk.make_plan(130, 8, 256, 8)["variant"] == 3      # one k-block: nothing to split
    p = tk.make_plan(300, 520, 40, 3)                        # 9 k-blocks: cluster capped at 8
    assert p["variant"] == 2 and p["cluster"] == 8


def test_plan_tmem_and_smem_budget():
    for T in (1, 1000, 30000):
        for E in range(16, 1025, 8):
            p = tk.make_plan(T, 7168, E, min(8, E), 148)
            assert p["expert_groups"] == (2 if p["n_pad"] > 512 else 1)
            acc = (min(p["n_pad"], 512) + 31) // 32 * 32
            # split-H keeps one accumulator; row tiles two, or one when two do not fit
            buffers = 1 if p["variant"] == 2 or 2 * acc > 512 else 2
            assert p["tmem_cols"] >= buffers * acc
            assert p["tmem_cols"] <= 512
            assert p["smem_bytes"] <= 232448
            assert p["stages"] >= 2 and p["slices_per_stage"] in (1, 2)
            if p["variant"] == 2:
                # the exchange stages 128 rows of up to 256 experts in the ring
                ring = p["smem_bytes"] - 1280
                row_stride = (min(E, 256) + 31) // 32 * 32 + 4
                assert 128 * row_stride * 4 <= ring


def test_plan_large_expert_counts():
    p = tk.make_plan(65536, 7168, 512, 8, 148)      # pairs, two 256-expert MMA chunks, one accumulator
    assert p["variant"] == 3 and p["n_pad"] == 512 and p["tmem_cols"] == 512
    p = tk.make_plan(65536, 7168, 320, 8, 148)      # 384 columns: chunks of 256 and 128
    assert p["variant"] == 3 and p["n_pad"] == 384 and p["tmem_cols"] == 512
    p = tk.make_plan(4096, 7168, 512, 32, 148)      # split-H, one 80 KB K slice per stage
    assert p["variant"] == 2 and p["slices_per_stage"] == 1 and p["tmem_cols"] == 512
    p = tk.make_plan(4096, 7168, 256, 8, 148)      # split-H: one K slice per ring stage
    assert p["slices_per_stage"] == 1 and p["stages"] == 4
    p = tk.make_plan(65536, 7168, 1024, 8, 148)     # two expert groups of 512, one after the other
    assert p["variant"] == 3 and p["n_pad"] == 1024 and p["expert_groups"] == 2 and p["tmem_cols"] == 512
    p = tk.make_plan(1, 7168, 1000, 8, 148)
    assert p["variant"] == 2 and p["expert_groups"] == 2 and p["tmem_cols"] == 512


def test_fp8_entry_point_rejects_before_cuda():
    f = tk.fused_topk_gating_fp8_ptr
    assert f(16, 16, 16, 16, 8, 72, 16, 2, 16, 16) == tk.TK_ERR_UNSUPPORTED        # H % 16 != 0
    assert f(16, 16, 16, 16, 8, 64, 16, 17, 16, 16) == tk.TK_ERR_INVALID_ARG       # k > E
    assert f(16, 16, 16, 16, 8, 64, 1032, 2, 16, 16) == tk.TK_ERR_UNSUPPORTED      # E > 1024
    assert f(16, 0, 16, 16, 8, 64, 16, 2, 16, 16) == tk.TK_ERR_INVALID_ARG         # null scale
    assert f(16, 20, 16, 16, 8, 64, 16, 2, 16, 16) == tk.TK_ERR_ALIGNMENT          # scale not 16-byte aligned
    assert f(0, 0, 0, 0, 0, 64, 16, 2, 0, 0) == tk.TK_OK                             # T == 0


def _header_struct_fields(name):
    import re
    text = open(tk.exported_symbols.__globals__["HEADER"]).read()
    body = dict((n, b) for b, n in re.findall(r"typedef struct \{([^}]*)\}\s*(\w+);", text))[name]
    return [(t, n) for t, n in re.findall(r"^\s*(int32_t|int64_t)\s+(\w+);", body, re.M)]


@pytest.mark.parametrize("name,binding", [("tk_gating_plan", "_Plan"), ("tk_route_plan", "_RoutePlan")])
def test_binding_structs_match_the_header(name, binding):
    from moe_router_gating_b200 import _binding
    fields = getattr(_binding, binding)._fields_
    ctype = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64}
    assert [(n, ctype[t]) for t, n in _header_struct_fields(name)] == [(n, t) for n, t in fields]


def test_header_is_plain_c(tmp_path):
    # the C ABI must be usable from C: the header compiles as C99 on its own
    src = tmp_path / "use_header.c"
    src.write_text('#include "tk_gating.h"\n'
                   'int main(void) { tk_gating_plan p; tk_route_plan q; (void)p; (void)q;\n'
                   '  return (int)sizeof(tk_status) + TK_GATING_MAX_EXPERTS + TK_ROUTE_STATIC_SCRATCH_BYTES; }\n')
    include = os.path.dirname(tk.exported_symbols.__globals__["HEADER"])
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-fsyntax-only", "-I", include, str(src)],
                   check=True)


@pytest.mark.parametrize("C", [2, 4, 8, 16])
@pytest.mark.parametrize("valid_rows", [1, 3, 31, 64, 100, 127, 128])
def test_split_h_staging_slots_are_distinct(C, valid_rows):
    # the exchange writes row t's partial from CTA r into owner t % C, slot (t / C) * C + r;
    # an owner reads its n_own rows at slots [s * C, s * C + C): every write lands once, in range
    n_own = {o: (valid_rows - o + C - 1) // C if valid_rows > o else 0 for o in range(C)}
    seen = set()
    for t in range(valid_rows):
        owner = t % C
        for r in range(C):
            slot = (t // C) * C + r
            assert 0 <= slot < n_own[owner] * C
            assert (owner, slot) not in seen
            seen.add((owner, slot))
    assert len(seen) == sum(n * C for n in n_own.values())


def test_logits_entry_points_reject_before_cuda():
    lib = tk.library()
    f = lib.tk_gating_fused_topk_logits
    assert f(16, 16, 8, 64, 16, 2, 16, 16, 0, 0) == tk.TK_ERR_INVALID_ARG      # null logits
    assert f(16, 16, 8, 64, 16, 2, 16, 16, 20, 0) == tk.TK_ERR_ALIGNMENT       # logits not 16-byte aligned
    assert f(16, 16, 8, 64, 20, 2, 16, 16, 0, 0) == tk.TK_ERR_UNSUPPORTED      # sizes are checked first
    assert f(0, 16, 8, 64, 16, 2, 16, 16, 16, 0) == tk.TK_ERR_INVALID_ARG      # null hidden
    assert f(0, 0, 0, 64, 16, 2, 0, 0, 0, 0) == tk.TK_OK                         # T == 0
    g = lib.tk_gating_fused_topk_fp8_logits
    assert g(16, 16, 16, 16, 8, 64, 16, 2, 16, 16, 0, 0) == tk.TK_ERR_INVALID_ARG
    assert g(16, 16, 16, 16, 8, 64, 16, 2, 16, 16, 24, 0) == tk.TK_ERR_ALIGNMENT
    assert g(16, 16, 16, 16, 8, 72, 16, 2, 16, 16, 0, 0) == tk.TK_ERR_UNSUPPORTED  # H % 16
    assert g(0, 0, 0, 0, 0, 64, 16, 2, 0, 0, 0, 0) == tk.TK_OK


def test_clock_counters_reject_null_pointers():
    c = ctypes.c_uint64(0)
    lib = tk.library()
    assert lib.tk_gating_clock_counters(None, ctypes.byref(c), ctypes.byref(c), 0) == tk.TK_ERR_INVALID_ARG
    assert lib.tk_gating_clock_counters(ctypes.byref(c), ctypes.byref(c), None, 1) == tk.TK_ERR_INVALID_ARG


def test_binding_rejects_bad_logits_before_the_call():
    from moe_router_gating_b200 import _binding
    with pytest.raises(ValueError):
        _binding._check_logits(torch.empty((3, 4)), 3, 5, torch.device("cpu"))
    with pytest.raises(ValueError):
        _binding._check_logits(torch.empty((3, 4), dtype=torch.float64), 3, 4, torch.device("cpu"))
    _binding._check_logits(torch.empty((3, 4)), 3, 4, torch.device("cpu"))



def test_fused_route_entry_point_rejects_before_cuda():
    f = tk.fused_topk_gating_route_ptr
    # (hidden, gate, T, H, E, k, scores, ids, offsets, sorted_slots, slot_pos, workspace, workspace_bytes)
    ok = (16, 16, 8, 64, 16, 2, 16, 16, 16, 16, 16, 16, 1 << 20)

    def call(**kw):
        names = ("hidden", "gate", "T", "H", "E", "k", "scores", "ids", "offsets", "sorted_slots", "slot_pos",
                 "workspace", "workspace_bytes")
        args = dict(zip(names, ok))
        args.update(kw)
        return f(*(args[n] for n in names))

    assert call(k=17) == tk.TK_ERR_INVALID_ARG           # k > E
    assert call(E=1032) == tk.TK_ERR_UNSUPPORTED         # E > 1024
    assert call(H=60) == tk.TK_ERR_UNSUPPORTED           # H % 8 != 0
    assert call(T=1 << 28, k=8) == tk.TK_ERR_UNSUPPORTED  # T * k >= 2^31
    assert call(offsets=0) == tk.TK_ERR_INVALID_ARG
    assert call(sorted_slots=0) == tk.TK_ERR_INVALID_ARG
    assert call(hidden=0) == tk.TK_ERR_INVALID_ARG
    assert call(slot_pos=18) == tk.TK_ERR_ALIGNMENT      # routing outputs: 4-byte aligned
    assert call(ids=20) == tk.TK_ERR_ALIGNMENT           # gating outputs: 16-byte aligned
    # valid arguments without a GPU: no CPU fallback
    assert call() in (tk.TK_ERR_CUDA, tk.TK_ERR_UNSUPPORTED)


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (512, 8, 256), (513, 8, 256), (65536, 8, 256), (3001, 16, 1024),
                                   (12345, 7, 999)])
def test_fused_route_workspace_is_the_table_and_a_counter(T, k, E):
    p = tk.route_plan(T, k, E, 148)
    if p["ctas"] == 1:
        assert p["fused_workspace_bytes"] == 0
    else:
        assert p["fused_workspace_bytes"] == p["workspace_bytes"] + 16 == p["ctas"] * ((E + 3) // 4 * 4) * 4 + 16
        # a gating row's k <= 32 assignments cross at most one routing range boundary
        assert p["warp_slots"] * 32 >= 4096 >= k


@pytest.mark.parametrize("T,H,E,k", [(65536, 7168, 256, 8), (20000, 7168, 256, 8), (65533, 6144, 200, 6),
                                     (23000, 6144, 136, 1), (65536, 7168, 256, 4)])
def test_workspace_plan_splits_the_last_round(T, H, E, k):
    plain = tk.make_plan(T, H, E, k, 148)
    plan, nbytes = tk.make_plan_ws(T, H, E, k, 148)
    assert plain["num_half_tiles"] > 0 and plan["num_half_tiles"] == 0
    n = plan["num_split_tiles"]
    assert n == (plain["num_half_tiles"] + 1) // 2 and 2 * n <= plan["grid"] // 2
    # every row is covered once: full tiles, then the split tiles (the last may run past T)
    assert plan["num_tiles"] * 256 < T <= (plan["num_tiles"] + n) * 256
    kb = plan["split_k_block"]
    assert kb % 2 == 0 and 0 < kb < plan["k_blocks"]
    cols = (E + 31) // 32 * 32
    assert nbytes == (n * 8 + 255) // 256 * 256 + n * 256 * (cols + 4) * 4
    # the first half's 128 rows of a CTA fit its ring once the ring is idle
    ring = plan["smem_bytes"] - 1280
    assert 128 * (cols + 4) * 4 <= ring
    for key in ("variant", "block_m", "n_pad", "k_blocks", "stages", "grid", "cluster", "threads", "smem_bytes"):
        assert plan[key] == plain[key], key


@pytest.mark.parametrize("T,H,E,k", [(4096, 7168, 256, 8), (65536, 4096, 256, 8), (65536, 7168, 512, 8),
                                     (60000, 4096, 256, 16), (16384, 4096, 64, 6), (5, 7168, 256, 8),
                                     (8, 7168, 256, 8), (1, 7168, 512, 8)])
def test_workspace_plan_elsewhere_is_the_plain_plan(T, H, E, k):
    assert tk.make_plan_ws(T, H, E, k, 148) == (tk.make_plan(T, H, E, k, 148), 0)


@pytest.mark.parametrize("num_sms", [148, 132, 16])
@pytest.mark.parametrize("T,H,E,k", [(1, 7168, 256, 8), (4, 7168, 256, 8), (3, 4096, 64, 6), (4, 512, 16, 2),
                                     (3, 2048, 200, 8), (2, 1000, 96, 16), (1, 8, 16, 4), (4, 7168, 256, 32)])
def test_workspace_plan_few_tokens(T, H, E, k, num_sms):
    plan, nbytes = tk.make_plan_ws(T, H, E, k, num_sms)
    assert plan["variant"] == 4 and plan["block_m"] == T and plan["cluster"] == 1 and plan["threads"] == 256
    e_blocks = (E + 31) // 32
    hb, rows = plan["split_h"], plan["h_rows"]
    assert plan["n_pad"] == 32 * e_blocks and plan["grid"] == hb * e_blocks <= max(num_sms, e_blocks)
    # the H ranges: multiples of 8 rows, none empty, covering H once
    assert rows % 8 == 0 and (hb - 1) * rows < H <= hb * rows
    # the counter (256 bytes), then h_blocks x T partial rows of n_pad floats
    assert nbytes == 256 + hb * T * plan["n_pad"] * 4
    # shared memory: barrier and flag, staged hidden values, the warps' sums, the copied partials, the sums
    def up(v):
        return (v + 127) // 128 * 128
    smem = 128 + up(T * rows * 4) + 8 * T * 32 * 4 + up(hb * T * plan["n_pad"] * 4) + T * plan["n_pad"] * 4
    assert plan["smem_bytes"] == smem <= 232448
    # the FP8 entry point keeps its plain plan
    if H % 16 == 0:
        assert tk.make_plan_ws(T, H, E, k, num_sms, fp8=True) == (tk.make_plan(T, H // 2, E, k, num_sms), 0)


def test_workspace_entry_points_reject_before_cuda():
    f = tk.fused_topk_gating_ws_ptr
    assert f(16, 16, 8, 64, 16, 17, 16, 16, 16, 1 << 20) == tk.TK_ERR_INVALID_ARG   # k > E
    assert f(16, 16, 8, 60, 16, 2, 16, 16, 16, 1 << 20) == tk.TK_ERR_UNSUPPORTED    # H % 8
    assert f(16, 16, 8, 64, 16, 2, 16, 16, 16, -1) == tk.TK_ERR_INVALID_ARG         # negative size
    assert f(0, 16, 8, 64, 16, 2, 16, 16, 16, 1 << 20) == tk.TK_ERR_INVALID_ARG     # null hidden
    assert f(16, 16, 8, 64, 16, 2, 20, 16, 16, 1 << 20) == tk.TK_ERR_ALIGNMENT      # scores
    assert f(0, 0, 0, 64, 16, 2, 0, 0, 0, 0) == tk.TK_OK                             # T == 0
    # valid arguments without a GPU: no CPU fallback
    assert f(16, 16, 65536, 7168, 256, 8, 16, 16, 16, 1 << 24) in (tk.TK_ERR_CUDA, tk.TK_ERR_UNSUPPORTED)
    lib = tk.library()
    n = ctypes.c_int64(-1)
    assert lib.tk_gating_workspace_bytes(8, 7168, 256, 8, 0, None) == tk.TK_ERR_INVALID_ARG
    assert lib.tk_gating_workspace_bytes(8, 60, 256, 8, 0, ctypes.byref(n)) == tk.TK_ERR_UNSUPPORTED
    assert lib.tk_gating_workspace_bytes(8, 7168, 256, 8, 1, ctypes.byref(n)) in (tk.TK_ERR_CUDA,
                                                                                   tk.TK_ERR_UNSUPPORTED)
    assert lib.tk_gating_fused_topk_fp8_ws(16, 16, 16, 16, 8, 72, 16, 2, 16, 16, 16, 1 << 20, None) == \
        tk.TK_ERR_UNSUPPORTED                                                          # FP8: H % 16 != 0
