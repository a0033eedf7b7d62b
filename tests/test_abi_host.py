"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe.h declares, and rejects bad arguments before it
touches the device (the counterpart of the ValueError the Mixtral textbook
page's MoE constructor raises for top_k_experts outside 1..num_experts,
sections "Mixtral" and "Конфигурация")."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    declared = _declared()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(binding.EXPORTS)


def test_status_strings():
    for code in range(6):
        assert binding.status_string(code).startswith("MOE_")


@pytest.mark.parametrize("shape,code", [
    ((64, 128, 256, 8, 2), moe.MOE_OK),
    ((0, 128, 256, 8, 2), moe.MOE_OK),
    ((64, 128, 256, 8, 0), moe.MOE_ERR_INVALID_ARG),   # k outside 1..E
    ((64, 128, 256, 8, 9), moe.MOE_ERR_INVALID_ARG),
    ((-1, 128, 256, 8, 2), moe.MOE_ERR_INVALID_ARG),
    ((64, 100, 256, 8, 2), moe.MOE_ERR_UNSUPPORTED),   # d not a multiple of 128
    ((64, 128, 200, 8, 2), moe.MOE_ERR_UNSUPPORTED),
    ((64, 128, 256, 33, 2), moe.MOE_ERR_UNSUPPORTED),  # E > 32
    ((64, 128, 256, 16, 9), moe.MOE_ERR_UNSUPPORTED),  # k > 8
    ((16, 4096, 14336, 32, 2), moe.MOE_ERR_UNSUPPORTED),  # router tile too large
    ((1 << 20, 4096, 14336, 8, 2), moe.MOE_ERR_UNSUPPORTED),  # 32-bit row index overflow
])
def test_shape_checks(shape, code):
    assert moe.moe_check_shape(shape) == code


def test_workspace_sizes():
    s = (4096, 4096, 14336, 8, 2)
    fwd = moe.moe_forward_workspace_bytes(s)
    R = 4096 * 2
    assert fwd >= R * 4096 * 2 + R * 14336 * 2 + R * 4096 * 4
    assert moe.moe_forward_hostio_workspace_bytes(s) == fwd + 2 * 4096 * 4096 * 2
    assert moe.moe_expert_workspace_bytes(s) >= 4
    assert moe.moe_forward_workspace_bytes((64, 128, 256, 8, 9)) == 0
    # decode batches of the Mixtral shape fit the static scratch, larger ones do not
    assert moe.moe_forward_workspace_bytes((64, 4096, 14336, 8, 2)) <= binding.MOE_STATIC_SCRATCH_BYTES
    assert moe.moe_forward_workspace_bytes((80, 4096, 14336, 8, 2)) > binding.MOE_STATIC_SCRATCH_BYTES


def test_forward_kernel_count():
    """Six kernels, five once the down projection forms y itself (4 or more
    rounds of its CTA-pair tiles; the host without a GPU assumes the B200's
    148 SMs, 74 pairs), none for an empty batch, an error for a rejected shape."""
    assert moe.moe_forward_kernel_count((4096, 4096, 14336, 8, 2)) == 5    # 512 pair tiles
    assert moe.moe_forward_kernel_count((1024, 1024, 3584, 8, 2)) == 6     # 32 pair tiles
    assert moe.moe_forward_kernel_count((16, 4096, 14336, 8, 2)) == 6      # single CTAs
    assert moe.moe_forward_kernel_count((16384, 4096, 14336, 8, 2)) == 5   # 2048 pair tiles
    assert moe.moe_forward_kernel_count((50600, 384, 256, 8, 2)) == 6      # d not a multiple of 256
    assert moe.moe_forward_kernel_count((0, 128, 256, 8, 2)) == 0
    with pytest.raises(moe.MoeError):
        moe.moe_forward_kernel_count((64, 128, 256, 8, 9))
    assert binding.lib().moe_forward_kernel_count(binding.MoeShape(64, 100, 256, 8, 2)) == \
        -moe.MOE_ERR_UNSUPPORTED


def _call(fn, *args):
    return getattr(binding.lib(), fn)(*args)


def test_null_and_misaligned_pointers_are_rejected_without_launch():
    S = binding.MoeShape(64, 128, 256, 8, 2)
    P = ctypes.c_void_p
    good = P(1 << 20)          # never dereferenced: validation fails first
    bad = P((1 << 20) + 8)     # not 16-byte aligned
    assert _call("moe_route", S, None, good, None, good, good, None, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_route", S, bad, good, None, good, good, None, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_combine", S, good, None, good, good, None) == moe.MOE_ERR_INVALID_ARG
    # every call below carries one invalid argument, so nothing may reach the device
    assert _call("moe_expert_swiglu", S, good, good, good, good, good, None, good, good,
                 ctypes.c_size_t(1 << 20), None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_expert_swiglu", S, good, good, good, good, good, good, good, good,
                 ctypes.c_size_t(16), None) == moe.MOE_ERR_WORKSPACE
    assert _call("moe_forward", S, good, good, None, good, good, good, good, None, None, good,
                 ctypes.c_size_t(16), None) == moe.MOE_ERR_WORKSPACE
    bad_k = binding.MoeShape(64, 128, 256, 8, 9)
    assert _call("moe_forward", bad_k, good, good, None, good, good, good, good, None, None, good,
                 ctypes.c_size_t(1 << 30), None) == moe.MOE_ERR_INVALID_ARG
    big = (1024, 1024, 3584, 8, 2)
    assert moe.moe_forward_workspace_bytes(big) > binding.MOE_STATIC_SCRATCH_BYTES
    assert _call("moe_forward_static", binding.MoeShape(*big), good, good, None,
                 good, good, good, good, None, None) == moe.MOE_ERR_WORKSPACE
    assert _call("moe_forward_profiled", S, good, good, None, good, good, good, good, good,
                 ctypes.c_size_t(1 << 30), None, 7, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_expert_swiglu_stall_test", S, good, good, good, good, good, good, good,
                 good, ctypes.c_size_t(1 << 20), -1, ctypes.c_uint64(10 ** 6),
                 None) == moe.MOE_ERR_INVALID_ARG
    # biased variants: a misaligned bias, then a short workspace
    assert _call("moe_expert_swiglu_bias", S, good, good, good, good, good, good, bad, None,
                 good, good, good, ctypes.c_size_t(1 << 20), None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_expert_swiglu_bias", S, good, good, good, good, good, None, None, None,
                 good, good, good, ctypes.c_size_t(16), None) == moe.MOE_ERR_WORKSPACE
    assert _call("moe_forward_bias", S, good, good, None, good, good, good, bad, good, good, good,
                 None, None, good, ctypes.c_size_t(1 << 30), None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_forward_bias", S, good, good, None, good, good, good, good, good, good, good,
                 None, None, good, ctypes.c_size_t(16), None) == moe.MOE_ERR_WORKSPACE


def test_block_hostio_and_dispatch_reject_bad_arguments_on_host():
    S = binding.MoeShape(64, 128, 256, 8, 2)
    P = ctypes.c_void_p
    good = P(1 << 20)
    bad = P((1 << 20) + 8)
    eps = ctypes.c_float(1e-5)
    big = ctypes.c_size_t(1 << 30)
    # block: a misaligned gamma, a negative eps, a NaN eps, a short workspace
    assert _call("moe_block_forward", S, good, bad, eps, good, None, good, good, good, good, good,
                 big, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_block_forward", S, good, good, ctypes.c_float(-1.0), good, None, good, good,
                 good, good, good, big, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_block_forward", S, good, good, ctypes.c_float(float("nan")), good, None,
                 good, good, good, good, good, big, None) == moe.MOE_ERR_INVALID_ARG
    need = moe.moe_block_workspace_bytes((64, 128, 256, 8, 2))
    assert _call("moe_block_forward", S, good, good, eps, good, None, good, good, good, good, good,
                 ctypes.c_size_t(need - 1), None) == moe.MOE_ERR_WORKSPACE
    # host I/O: missing host buffers, then a workspace one byte short
    assert _call("moe_forward_hostio", S, None, good, None, good, good, good, good, good, big,
                 None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_forward_hostio", S, good, good, None, good, good, good, None, good, big,
                 None) == moe.MOE_ERR_INVALID_ARG
    need = moe.moe_forward_hostio_workspace_bytes((64, 128, 256, 8, 2))
    assert _call("moe_forward_hostio", S, good, good, None, good, good, good, good, good,
                 ctypes.c_size_t(need - 1), None) == moe.MOE_ERR_WORKSPACE
    # dispatch: no offsets, a misaligned x
    assert _call("moe_dispatch", S, good, good, None, good, good, good, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert _call("moe_dispatch", S, good, bad, good, good, good, good, None) == \
        moe.MOE_ERR_INVALID_ARG


def test_hostio_stall_hook_rejects_bad_arguments_on_host():
    S = binding.MoeShape(64, 128, 256, 8, 2)
    P = ctypes.c_void_p
    good = P(1 << 20)
    big = ctypes.c_size_t(1 << 30)
    t = ctypes.c_uint64(10 ** 6)
    assert _call("moe_forward_hostio_stall_test", S, good, good, None, good, good, good, good,
                 good, big, -1, 1, t, None) == moe.MOE_ERR_INVALID_ARG      # negative chunk
    assert _call("moe_forward_hostio_stall_test", S, good, good, None, good, good, good, good,
                 good, big, 0, -1, t, None) == moe.MOE_ERR_INVALID_ARG      # negative stage count
    assert _call("moe_forward_hostio_stall_test", S, good, good, None, good, good, good, good,
                 good, big, 0, 1, ctypes.c_uint64(10), None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_forward_hostio_stall_test", S, None, good, None, good, good, good, good,
                 good, big, 0, 1, t, None) == moe.MOE_ERR_INVALID_ARG      # no host x


def test_static_scratch_limit_is_78_tokens_at_the_mixtral_widths():
    """The static scratch holds the whole forward workspace of up to 78 tokens
    at d = 4096, d_ff = 14336, k = 2; 79 tokens are rejected before any launch."""
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert moe.moe_forward_workspace_bytes((78, 4096, 14336, 8, 2)) <= binding.MOE_STATIC_SCRATCH_BYTES
    assert moe.moe_forward_workspace_bytes((79, 4096, 14336, 8, 2)) > binding.MOE_STATIC_SCRATCH_BYTES
    assert _call("moe_forward_static", binding.MoeShape(79, 4096, 14336, 8, 2), good, good, None,
                 good, good, good, good, None, None) == moe.MOE_ERR_WORKSPACE
    # T = 0 launches nothing (no status pointer given)
    assert _call("moe_forward_static", binding.MoeShape(0, 4096, 14336, 8, 2), None, None, None,
                 None, None, None, None, None, None) == moe.MOE_OK


def test_aux_loss_rejects_bad_arguments_on_host():
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert _call("moe_aux_loss", binding.MoeShape(16, 128, 256, 8, 9), good, good, None, good,
                 None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_aux_loss", binding.MoeShape(16, 128, 256, 8, 2), good, good, None, None,
                 None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert _call("moe_aux_loss", binding.MoeShape(16, 128, 256, 64, 2), good, good, None, good,
                 None, None, None) == moe.MOE_ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op_on_host():
    S = binding.MoeShape(0, 128, 256, 8, 2)
    for fn, nargs in (("moe_route", 7), ("moe_combine", 5)):
        assert _call(fn, S, *([None] * nargs)) == moe.MOE_OK


def test_hostio_batches_rejects_bad_arguments_on_host():
    S = binding.MoeShape(64, 128, 256, 8, 2)
    P = ctypes.c_void_p
    good = P(1 << 20)
    arr = (P * 2)(1 << 20, 1 << 21)
    holey = (P * 2)(1 << 20, None)
    big = ctypes.c_size_t(1 << 30)
    fn = "moe_forward_hostio_batches"
    assert _call(fn, S, 0, arr, good, None, good, good, good, arr, good, big, None) == \
        moe.MOE_ERR_INVALID_ARG                                         # no batches
    assert _call(fn, S, 2, None, good, None, good, good, good, arr, good, big, None) == \
        moe.MOE_ERR_INVALID_ARG                                         # no x array
    assert _call(fn, S, 2, arr, good, None, good, good, good, holey, good, big, None) == \
        moe.MOE_ERR_INVALID_ARG                                         # a null y entry
    need = moe.moe_forward_hostio_batches_workspace_bytes((64, 128, 256, 8, 2))
    # small batches: a forward workspace for each of two compute streams
    assert need == 2 * moe.moe_forward_workspace_bytes((64, 128, 256, 8, 2)) + 4 * 64 * 128 * 2
    large = (4096, 4096, 14336, 8, 2)  # one compute stream
    assert moe.moe_forward_hostio_batches_workspace_bytes(large) == \
        moe.moe_forward_workspace_bytes(large) + 4 * 4096 * 4096 * 2
    assert _call(fn, S, 2, arr, good, None, good, good, good, arr, good,
                 ctypes.c_size_t(need - 1), None) == moe.MOE_ERR_WORKSPACE
    # T = 0 enqueues nothing
    assert _call(fn, binding.MoeShape(0, 128, 256, 8, 2), 2, arr, None, None, None, None, None,
                 arr, None, ctypes.c_size_t(0), None) == moe.MOE_OK


def test_hostio_batches_stall_hook_rejects_bad_arguments_on_host():
    S = binding.MoeShape(64, 128, 256, 8, 2)
    P = ctypes.c_void_p
    good = P(1 << 20)
    arr = (P * 2)(1 << 20, 1 << 21)
    big = ctypes.c_size_t(1 << 30)
    t = ctypes.c_uint64(10 ** 6)
    fn = "moe_forward_hostio_batches_stall_test"
    assert _call(fn, S, 2, arr, good, None, good, good, good, arr, good, big, -1, 1, t,
                 None) == moe.MOE_ERR_INVALID_ARG                          # negative batch
    assert _call(fn, S, 2, arr, good, None, good, good, good, arr, good, big, 0, -1, t,
                 None) == moe.MOE_ERR_INVALID_ARG                          # negative stage count
    assert _call(fn, S, 2, arr, good, None, good, good, good, arr, good, big, 0, 1,
                 ctypes.c_uint64(10), None) == moe.MOE_ERR_INVALID_ARG     # timeout too short
    assert _call(fn, S, 0, arr, good, None, good, good, good, arr, good, big, 0, 1, t,
                 None) == moe.MOE_ERR_INVALID_ARG                          # no batches
