"""The C-ABI library loads, exports every entry point of include/w4a8.h, and
rejects bad arguments on the host (no CUDA work is done; runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")


@pytest.fixture(scope="module")
def L():
    from w4a8_quantized_moe_b200 import build as b
    b.build()
    import w4a8_quantized_moe_b200 as m
    return m.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a8_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["w4a8_pack_int4", "w4a8_quant_act_fp8_per_token", "w4a8_moe_route_permute",
                 "w4a8_moe_forward", "w4a8_moe_workspace_size", "w4a8_check_device_error"]:
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} is declared in w4a8.h but not exported"


def test_library_exports_nothing_else(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("nm not available")
    exported = {ln.split()[-1] for ln in out.stdout.splitlines() if " T " in ln}
    ours = {n for n in exported if n.startswith("w4a8_")}
    assert ours == set(declared_functions())


def test_status_strings_and_version(L):
    assert L.w4a8_abi_version() == 1
    assert L.w4a8_status_string(0) == b"W4A8_OK"
    assert L.w4a8_status_string(6) == b"W4A8_ERR_DEVICE_TIMEOUT"
    assert L.w4a8_status_string(7) == b"W4A8_ERR_DEVICE_INDEX"
    assert L.w4a8_status_string(99) == b"W4A8_ERR_UNKNOWN"


def test_release_and_bounds_checking_builds():
    # the two builds of the same sources: same exports, and the build flag
    # tells them apart (the debug build checks routing-derived indices)
    from w4a8_quantized_moe_b200 import build as b
    rel = ctypes.CDLL(b.build())
    dbg = ctypes.CDLL(b.build(debug_bounds=True))
    assert rel.w4a8_build_flags() == 0
    assert dbg.w4a8_build_flags() == 1
    for name in declared_functions():
        assert hasattr(dbg, name), f"{name} missing from the debug build"


def test_workspace_sizes_are_host_arithmetic(L):
    small = L.w4a8_moe_workspace_size(16, 512, 256, 8, 2)
    big = L.w4a8_moe_workspace_size(64, 6144, 2048, 256, 8)
    assert 0 < small < big
    A, H, I = 64 * 8, 6144, 2048
    # at least h (fp32), the intermediate codes and Y (fp32)
    assert big >= A * I * 4 + A * I + A * H * 4
    assert L.w4a8_moe_workspace_size(-1, 512, 256, 8, 2) == 0
    assert L.w4a8_moe_route_workspace_size(65536, 256) >= 2 * 256 * 256 * 4


def test_host_validation_without_device(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: validation fails first
    # group must be 128
    assert L.w4a8_pack_int4(fake, 4, 256, 64, fake, fake, None) == 2
    # K must be a multiple of 128
    assert L.w4a8_pack_int4(fake, 4, 200, 128, fake, fake, None) == 2
    assert b"multiple of 128" in L.w4a8_last_error()
    # empty input is a no-op that succeeds without touching the device
    assert L.w4a8_pack_int4(None, 0, 256, 128, None, None, None) == 0
    assert L.w4a8_quant_act_fp8_per_token(fake, -1, 128, fake, fake, None) == 1
    assert L.w4a8_quant_act_fp8_per_token(fake, 4, 100, fake, fake, None) == 2
    assert L.w4a8_quant_act_fp8_per_token(None, 0, 128, None, None, None) == 0
    # routing limits
    assert L.w4a8_moe_route_permute(fake, 4, 2000, 2, fake, fake, fake, fake, fake, fake, 1 << 30,
                                    None) == 2
    assert L.w4a8_moe_route_permute(fake, 4, 8, 9, fake, fake, fake, fake, fake, fake, 1 << 30,
                                    None) == 2
    assert L.w4a8_moe_route_permute(fake, 4, 64, 33, fake, fake, fake, fake, fake, fake, 1 << 30,
                                    None) == 2
    # misaligned pointer
    assert L.w4a8_moe_route_permute(vp((1 << 20) + 4), 4, 8, 2, fake, fake, fake, fake, fake,
                                    fake, 1 << 30, None) == 1
    # workspace too small
    assert L.w4a8_moe_route_permute(fake, 300, 8, 2, fake, fake, fake, fake, fake, fake, 16,
                                    None) == 4
    args = [fake, fake, fake, fake, fake, fake]
    # H not a multiple of 128
    assert L.w4a8_moe_forward(*args, 4, 200, 256, 8, 2, fake, fake, 1 << 40, None, None) == 2
    # I not a multiple of 128
    assert L.w4a8_moe_forward(*args, 4, 256, 100, 8, 2, fake, fake, 1 << 40, None, None) == 2
    # NULL weight
    assert L.w4a8_moe_forward(fake, fake, None, fake, fake, fake, 4, 256, 256, 8, 2, fake, fake,
                              1 << 40, None, None) == 1
    # short workspace
    assert L.w4a8_moe_forward(*args, 4, 256, 256, 8, 2, fake, fake, 1024, None, None) == 4
    # T == 0 is a no-op
    assert L.w4a8_moe_forward(None, None, None, None, None, None, 0, 256, 256, 8, 2, None, None, 0,
                              None, None) == 0
    # all-to-all dispatch: rank count, send-list capacity, shapes
    assert L.w4a8_ep_dispatch_plan(fake, 4, 2, 8, 65, fake, fake, 8, fake, None) == 2
    assert L.w4a8_ep_dispatch_plan(fake, 4, 2, 8, 0, fake, fake, 8, fake, None) == 2
    assert L.w4a8_ep_dispatch_plan(fake, 4, 2, 8, 4, fake, fake, 7, fake, None) == 1
    assert b"capacity" in L.w4a8_last_error()
    assert L.w4a8_ep_dispatch_plan(fake, 4, 0, 8, 4, fake, fake, 8, fake, None) == 1
    assert L.w4a8_ep_gather_rows(fake, fake, fake, fake, 4, 200, 2, fake, 3, fake, fake, fake,
                                 fake, None) == 2
    assert L.w4a8_ep_gather_rows(None, None, None, None, 4, 256, 2, None, 0, None, None, None,
                                 None, None) == 0
    assert L.w4a8_ep_combine_rows(fake, 3, 100, fake, 4, 2, fake, None) == 2
    assert L.w4a8_ep_combine_rows(fake, 3, 256, fake, 4, 65, fake, None) == 2
    assert L.w4a8_ep_combine_rows(None, 0, 256, None, 0, 2, None, None) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    import w4a8_quantized_moe_b200 as m
    with pytest.raises(ValueError, match="CUDA"):
        m.w4a8_quant_act_fp8_per_token(torch.zeros(4, 128, dtype=torch.bfloat16))


def test_shared_expert_entries_validate_on_the_host(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    # block quantiser: both dimensions multiples of 128
    assert L.w4a8_quant_fp8_block(fake, 100, 128, fake, fake, None) == 2
    assert L.w4a8_quant_fp8_block(fake, 128, 200, fake, fake, None) == 2
    assert L.w4a8_quant_fp8_block(None, 0, 128, None, None, None) == 0
    assert L.w4a8_quant_fp8_block(vp((1 << 20) + 8), 128, 128, fake, fake, None) == 1
    # group activation quantiser
    assert L.w4a8_quant_act_fp8_group(fake, -1, 128, fake, fake, None) == 1
    assert L.w4a8_quant_act_fp8_group(fake, 4, 100, fake, fake, None) == 2
    assert L.w4a8_quant_act_fp8_group(None, 0, 128, None, None, None) == 0
    # workspace sizes: host arithmetic, the combined layer needs both parts
    T, H, I = 64, 6144, 2048
    ws = L.w4a8_shared_expert_workspace_size(T, H, I)
    assert ws >= T * H + T * (H // 128) * 4 + T * I * 4 + T * I + T * (I // 128) * 4
    assert L.w4a8_shared_expert_workspace_size(-1, H, I) == 0
    both = L.w4a8_moe_shared_workspace_size(T, H, I, 256, 8, I)
    assert both >= L.w4a8_moe_workspace_size(T, H, I, 256, 8) + ws + T * H * 4 - 4096
    # the expert alone: shapes, NULL, workspace, empty input
    w = [fake] * 5
    assert L.w4a8_shared_expert_forward(*w, 4, 256, 100, fake, fake, 1 << 40, None, None) == 2
    assert L.w4a8_shared_expert_forward(*w, 4, 200, 128, fake, fake, 1 << 40, None, None) == 2
    assert L.w4a8_shared_expert_forward(fake, None, fake, fake, fake, 4, 256, 128, fake, fake,
                                        1 << 40, None, None) == 1
    assert L.w4a8_shared_expert_forward(*w, 4, 256, 128, fake, fake, 64, None, None) == 4
    assert L.w4a8_shared_expert_forward(None, None, None, None, None, 0, 256, 128, None, None, 0,
                                        None, None) == 0
    # the combined layer: the shared expert's width is checked, and its weights
    routed = [fake] * 6
    shared = [fake] * 4
    assert L.w4a8_moe_forward_shared(*routed, *shared, 4, 256, 256, 100, 8, 2, fake, fake,
                                     1 << 40, None, None, None) == 2
    assert L.w4a8_moe_forward_shared(*routed, None, fake, fake, fake, 4, 256, 256, 128, 8, 2,
                                     fake, fake, 1 << 40, None, None, None) == 1
    assert L.w4a8_moe_forward_shared(*routed, *shared, 4, 256, 256, 128, 8, 2, fake, fake, 1024,
                                     None, None, None) == 4


def test_binding_checks_shared_expert_arguments_before_any_cuda_call():
    import torch
    import w4a8_quantized_moe_b200 as m
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        m.w4a8_quant_fp8_block(torch.zeros(128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        m.w4a8_quant_act_fp8_group(x)
    w13c = torch.zeros(256, 256, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        m.w4a8_shared_expert_forward(x, w13c, torch.zeros(2, 2), torch.zeros(256, 128,
                                     dtype=torch.uint8), torch.zeros(2, 1))
