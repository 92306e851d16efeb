"""The C-ABI library builds, loads without a GPU, and exports every entry
point include/moe.h declares.  No compute call is made here."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    lib = ctypes.CDLL(abi.LIB_PATH)
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(abi.EXPORTS) == names


def test_host_only_calls():
    from moe_expert_layer_replay_b200 import abi
    d = abi.dims(4096, 2048, 1024, 64, 6)
    assert abi.rows_capacity(d) == (4096 * 6 + 64 * 127 + 127) // 128 * 128
    assert abi.permute_workspace_size(d) > 0
    assert abi.strerror(abi.BAD_ROUTING).startswith("routing")
    # argument checks run before any device work
    for bad in [abi.dims(16, 200, 128, 8, 2), abi.dims(16, 256, 128, 300, 2), abi.dims(16, 256, 128, 8, 9)]:
        st = abi.lib().moe_route_topk(None, ctypes.byref(bad), None, None, None)
        assert st in (abi.INVALID_ARG, abi.UNSUPPORTED)
    g = abi.GemmArgs()
    assert abi.lib().moe_grouped_gemm_fp8(0, ctypes.byref(abi.dims(16, 256, 100, 8, 2)), None,
                                          ctypes.byref(g), None) == abi.UNSUPPORTED
    assert abi.lib().moe_grouped_gemm_fp8(0, ctypes.byref(abi.dims(16, 256, 128, 8, 2)), None,
                                          ctypes.byref(g), None) == abi.INVALID_ARG


def test_gemm_operand_contract():
    """Per-op operand requirements of moe_grouped_gemm_fp8 are checked on the
    host, before any device work: the SiLU-backward GEMM needs its bf16 output
    (its codes are made from it), both SiLU GEMMs 32-byte-aligned aux / bf16 outputs, and the wgrad GEMMs need 16-byte-aligned
    scale arrays (they are bulk-copied)."""
    from moe_expert_layer_replay_b200 import abi
    L = abi.lib()
    d = abi.dims(4096, 2048, 1024, 64, 6)
    A = 0x100000  # aligned stand-ins; never dereferenced, every call fails its checks first
    offs = ctypes.c_void_p(A)
    g = abi.GemmArgs(A, A, A, A, A, A, A, None, None)  # b2 without out_bf16
    assert L.moe_grouped_gemm_fp8(abi.GEMM_DGRAD_DOWN_SILU, ctypes.byref(d), offs, ctypes.byref(g), None) \
        == abi.INVALID_ARG
    # a6 (training outputs) and b2 move 32-byte pieces of aux, out_bf16 (and b2's
    # out_q): each must be 32-byte aligned
    for op, fields in ((abi.GEMM_DGRAD_DOWN_SILU, (4, 5, 7)), (abi.GEMM_GATEUP_SILU, (4, 7))):
        for i in fields:
            ptrs = [A] * 8 + [None]
            ptrs[i] = A + 16
            g = abi.GemmArgs(*ptrs)
            assert L.moe_grouped_gemm_fp8(op, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG
    for op in (abi.GEMM_WGRAD_DOWN, abi.GEMM_WGRAD_GATEUP):
        g = abi.GemmArgs(A, A + 4, A, A, None, None, None, None, A)  # sa only 4-byte aligned
        assert L.moe_grouped_gemm_fp8(op, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG
        g = abi.GemmArgs(A, A, A, A + 8, None, None, None, None, A)  # sb only 8-byte aligned
        assert L.moe_grouped_gemm_fp8(op, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG
        g = abi.GemmArgs(A, A, A, A, None, None, None, None, None)  # no dW
        assert L.moe_grouped_gemm_fp8(op, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG
    g = abi.GemmArgs(A, A, A, A, None, None, None, None, None)  # a7 without Y
    assert L.moe_grouped_gemm_fp8(abi.GEMM_DOWN, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG
    assert L.moe_grouped_gemm_fp8(9, ctypes.byref(d), offs, ctypes.byref(g), None) == abi.INVALID_ARG


def test_empty_batch_host_paths():
    """T = 0: the entry points that have nothing to do return OK before any
    device work, with the (empty, so NULL) arrays left unchecked."""
    from moe_expert_layer_replay_b200 import abi
    L = abi.lib()
    d = abi.dims(0, 256, 128, 8, 2)
    assert L.moe_route_replay(None, 4, 1, ctypes.byref(d), None, None, None, None, None) == abi.OK
    assert L.moe_combine(None, None, None, ctypes.byref(d), None, None) == abi.OK
    assert L.moe_unpermute_reduce(None, None, ctypes.byref(d), None, None) == abi.OK
    # the layer index is still checked
    assert L.moe_route_replay(None, 4, 4, ctypes.byref(d), None, None, None, None, None) == abi.INVALID_ARG
