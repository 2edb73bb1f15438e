"""kvs_decode_attn_static: the decode step for callers that cannot allocate device
memory when they call the library (fixed memory plans, enqueue-only plugin hosts,
code that must not let an allocation synchronise the device).

It must give what kvs_decode_attn gives with a caller-provided workspace, call
after call, while using only the library's built-in scratch buffer: after the first
call on a device (the set-up call), further calls leave the device's free memory and
torch's allocations unchanged. A head already at capacity cannot take the appended
row; both entry points must report that, the static one through
kvs_static_device_flags. This file is collected last so that a run that stops at its
first failure has already run every other test; it also passes when run alone in a
fresh process.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from asymmetric_kv_merging_b200 import build
    build.build()
    from asymmetric_kv_merging_b200 import kvs as mod
    return mod


@pytest.mark.parametrize("dtype,d,G", [(torch.bfloat16, 128, 4), (torch.float32, 64, 2)])
def test_static_scratch_decode_matches_workspace_decode(kvs, dtype, d, G):
    dev = torch.device("cuda")
    B, H, T_cap = 2, 4, 3000
    g = torch.Generator().manual_seed(11)
    K = torch.randn(B, H, T_cap, d, generator=g).to(dtype).to(dev)
    V = torch.randn(B, H, T_cap, d, generator=g).to(dtype).to(dev)
    logn = torch.log(torch.randint(1, 4, (B, H, T_cap), generator=g).float()).to(dev)
    # the last head is full: it cannot take the appended row
    lens = torch.tensor([2500, 17, 0, 999, 1024, 2047, 64, T_cap], dtype=torch.int32, device=dev)
    desc = kvs.make_desc(B, H, H * G, d, T_cap, dtype)
    ws = kvs.workspace(desc, 32, ops=(kvs.OP_DECODE,))
    # two identical caches: one advanced by kvs_decode_attn, one by the static variant
    Ka, Va, La, la = K.clone(), V.clone(), logn.clone(), lens.clone()
    Kb, Vb, Lb, lb = K.clone(), V.clone(), logn.clone(), lens.clone()
    out_a = torch.empty(B, H * G, d, dtype=dtype, device=dev)
    out_b = torch.empty_like(out_a)
    steps = 3
    qs = [(torch.randn(B, H * G, d, generator=g) * 2).to(dtype).to(dev) for _ in range(steps)]
    kns = [torch.randn(B, H, d, generator=g).to(dtype).to(dev) for _ in range(steps)]
    vns = [torch.randn(B, H, d, generator=g).to(dtype).to(dev) for _ in range(steps)]
    torch.cuda.synchronize()
    kvs.static_device_flags(clear=True)          # set-up call: module load, address look-up
    mem = None
    for step in range(steps):
        kvs.decode_attn(desc, qs[step], Ka, Va, La, la, out_a, ws, kns[step], vns[step])
        kvs.decode_attn_static(desc, qs[step], Kb, Vb, Lb, lb, out_b, kns[step], vns[step])
        torch.cuda.synchronize()
        now = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated())
        if step >= 1:       # calls after the first allocate nothing
            assert now == mem, (now, mem)
        mem = now
        tol = dict(rtol=2e-2, atol=1e-2) if dtype == torch.bfloat16 else dict(rtol=1e-4, atol=1e-4)
        torch.testing.assert_close(out_b.float(), out_a.float(), **tol)
        assert torch.equal(lb, la)
        assert torch.equal(Kb, Ka) and torch.equal(Vb, Va) and torch.equal(Lb, La)
        # both report the full head, every step; the static flags accumulate until read
        assert kvs.device_flags(ws, clear=True) == kvs.FLAG_OUT_CAPACITY
    expect = lens.cpu() + steps
    expect[-1] = T_cap                            # rejected append: length unchanged
    assert torch.equal(la.cpu(), expect)
    assert kvs.static_device_flags(clear=True) == kvs.FLAG_OUT_CAPACITY
    assert kvs.static_device_flags() == 0


def test_static_scratch_rejects_shapes_beyond_its_size(kvs):
    # 256 sequences x 8 KV heads x 8 query heads each: 16384 query heads of split
    # partials (about 8.5 MB) do not fit the 4 MiB buffer
    desc = kvs.make_desc(256, 8, 64, 128, 1024, kvs.BF16)
    assert kvs.workspace_size(desc, 0, kvs.OP_DECODE) > kvs.static_scratch_bytes()
    with pytest.raises(kvs.KvsError) as e:
        kvs.decode_attn_static(desc, None, None, None, None, None, None)
    assert e.value.status == 4          # KVS_ERR_WORKSPACE, nothing launched
