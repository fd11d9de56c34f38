"""The allocation-free entry point, pisa_attention_noalloc.

Callers that may not allocate device memory (a plugin whose host application
owns the whole device memory pool, or a loop where cudaMalloc/cudaFree are not
allowed) use this entry point; it takes its scratch from an array built into
the library instead of a caller workspace.  These tests call it through the C
ABI and check that it returns what pisa_attention returns, bit for bit (both
run the same deterministic kernels on the same inputs), on two calls in a row
(the second call finds the first call's data still in the shared scratch), and
that a call leaves the device's free memory and torch's allocation unchanged.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_taylor_b200 as pisa
import oracle
import pisa_synth

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def _c_noalloc(q, k, v, B, K, order, out):
    """Call pisa_attention_noalloc directly through ctypes."""
    lib = pisa.lib()
    fn = lib.pisa_attention_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 8 + [ctypes.c_void_p] * 2
    fn.restype = ctypes.c_int
    BH, L, d = q.shape
    code = pisa.PISA_BF16 if q.dtype == torch.bfloat16 else pisa.PISA_F32
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), 1, BH, L, d, code, B, K, order, out.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
@pytest.mark.parametrize("dt,d,B,order,L,BH", [(torch.bfloat16, 128, 64, 1, 4096, 4),
                                               (torch.bfloat16, 64, 64, 2, 2048, 3),
                                               (torch.float32, 64, 64, 1, 1024, 2)])
def test_noalloc_matches_pisa_attention_on_two_calls(dt, d, B, order, L, BH):
    K = (L // B) // 8
    for seed in (1, 2):  # two calls in a row through the same scratch
        q, k, v = (torch.from_numpy(x).to("cuda").to(dt) for x in
                   pisa_synth.random_qkv(900 + seed, BH, L, d, scale=2.0,
                                         dtype="bf16" if dt == torch.bfloat16 else "f32"))
        ref = pisa.pisa_attention(q, k, v, B, K, order)
        out = torch.full_like(q, float("nan"))
        assert _c_noalloc(q, k, v, B, K, order, out) == pisa.PISA_OK, pisa.lib().pisa_last_error()
        pisa.pisa_poll_device_status()
        assert torch.equal(out, ref)
        err = oracle.rel_l2(out.float().cpu().numpy(), ref.float().cpu().numpy())
        assert err <= TOL[dt], err


@pytest.mark.gpu
def test_noalloc_call_allocates_no_device_memory():
    # After a first call on the device (which resolves the scratch array's address and loads the
    # library's kernels), further calls change neither the device's free memory nor torch's
    # allocation.
    q, k, v = (torch.from_numpy(x).to("cuda").to(torch.bfloat16) for x in
               pisa_synth.random_qkv(950, 4, 4096, 128, scale=2.0, dtype="bf16"))
    out = torch.empty_like(q)
    assert _c_noalloc(q, k, v, 64, 8, 1, out) == pisa.PISA_OK, pisa.lib().pisa_last_error()
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        assert _c_noalloc(q, k, v, 64, 8, 1, out) == pisa.PISA_OK, pisa.lib().pisa_last_error()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0


@pytest.mark.gpu
def test_noalloc_rejects_calls_larger_than_its_scratch():
    lib = pisa.lib()
    lib.pisa_noalloc_scratch_bytes.restype = ctypes.c_size_t
    cap = lib.pisa_noalloc_scratch_bytes()
    assert cap == 32 << 20
    # 200 heads of the Wan shape need far more than the built-in scratch
    need = pisa.pisa_workspace_bytes(1, 200, 32768, 128, 64, 77, 1, torch.bfloat16)
    assert need > cap
    fn = lib.pisa_attention_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 8 + [ctypes.c_void_p] * 2
    fn.restype = ctypes.c_int
    fake = ctypes.c_void_p(0x1000)  # rejected before any pointer is used
    st = fn(fake, fake, fake, 1, 200, 32768, 128, pisa.PISA_BF16, 64, 77, 1, fake, None)
    assert st == pisa.PISA_ERR_INVALID_ARG
    assert b"scratch" in lib.pisa_last_error()
