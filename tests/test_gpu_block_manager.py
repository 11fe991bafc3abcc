"""GPU side of the block manager: pa_copy_blocks (the copy-on-write copies)
bit for bit, and a serving trace driven by the host manager -- prompts with
a shared prefix, a fork, decode steps with copy-on-write -- whose pool and
decode outputs match the CPU oracle run on the same operations."""

import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from tests.gpu_helpers import TOL, assert_close, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_device_errors():
    if torch.cuda.is_available():
        pa.device_errors()
    yield


@pytest.mark.parametrize("dtype,hkv,bs,d", [(torch.bfloat16, 8, 16, 128), (torch.bfloat16, 4, 128, 256),
                                            (torch.float32, 2, 16, 64)])
def test_copy_blocks_is_bit_exact(dtype, hkv, bs, d):
    g = torch.Generator(device="cuda").manual_seed(5)
    nb = 64
    kc = torch.randn((nb, hkv, bs, d), generator=g, device="cuda").to(dtype)
    vc = torch.randn((nb, hkv, bs, d), generator=g, device="cuda").to(dtype)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1))
    pairs = torch.stack([perm[:20], perm[20:40]], 1).to(torch.int32)  # disjoint sources and destinations
    kref, vref = kc.clone(), vc.clone()
    kref[pairs[:, 1].long()] = kc[pairs[:, 0].long()]
    vref[pairs[:, 1].long()] = vc[pairs[:, 0].long()]
    pa.copy_blocks(kc, vc, pairs.cuda())
    torch.cuda.synchronize()
    assert torch.equal(bits(kc), bits(kref)) and torch.equal(bits(vc), bits(vref))
    assert pa.device_errors() == 0


def test_copy_blocks_skips_ids_outside_the_pool():
    kc = torch.zeros((4, 1, 16, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[0] = 1.0
    pa.copy_blocks(kc, vc, torch.tensor([[0, 1], [0, 9], [-3, 2]], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert pa.device_errors() & pa.DEVERR_BLOCK
    assert (kc[1] == 1.0).all() and (kc[2] == 0).all() and (kc[3] == 0).all()


def test_manager_driven_trace_matches_the_oracle():
    torch.manual_seed(0)
    nb, bs, hkv, hq, d = 48, 16, 4, 16, 128
    m = pa.BlockManager(nb, bs)
    g = torch.Generator().manual_seed(3)
    kc = torch.full((nb, hkv, bs, d), float("nan"), dtype=torch.bfloat16)
    vc = torch.full_like(kc, float("nan"))
    kc_dev, vc_dev = kc.cuda(), vc.cuda()

    def write(slots, rows_k, rows_v):
        oracle.write_kv(rows_k, rows_v, slots, kc, vc)
        pa.write_kv(rows_k.cuda(), rows_v.cuda(), slots.cuda(), kc_dev, vc_dev)

    prefix = list(range(40))
    prompts = {1: prefix + [100, 101, 102], 2: prefix + [200], 3: [7, 7, 7, 7, 7]}
    for sid, toks in prompts.items():
        cached = m.add_sequence(sid, len(toks), toks)
        n_new = len(toks) - cached
        slots = m.slots(sid, cached, n_new)
        rows = torch.randn((n_new, hkv, d), generator=g).to(torch.bfloat16)
        write(slots, rows, rows * 0.5)
    assert m.add_sequence(4, 33, prefix[:33]) == 32  # two full blocks of the shared prefix are reused
    write(m.slots(4, 32, 1), torch.ones((1, hkv, d), dtype=torch.bfloat16), torch.ones((1, hkv, d),
                                                                                         dtype=torch.bfloat16))
    m.fork(1, 5)  # parallel sampling: 5 shares 1's blocks, including the partial last one
    seqs = [1, 2, 3, 4, 5]
    for step in range(20):
        slots, cow = m.append_slots(seqs, [step] * len(seqs))
        if cow.shape[0]:
            for s, t in cow.tolist():
                kc[t], vc[t] = kc[s], vc[s]
            pa.copy_blocks(kc_dev, vc_dev, cow.cuda())
        rows = torch.randn((len(seqs), hkv, d), generator=g).to(torch.bfloat16)
        write(slots, rows, -rows)
    torch.cuda.synchronize()
    assert torch.equal(bits(kc_dev), bits(kc)) and torch.equal(bits(vc_dev), bits(vc))

    tables, lens = m.block_tables(seqs, 8)
    q = torch.randn((len(seqs), hq, d), generator=g).to(torch.bfloat16)
    out = pa.decode_splitk(q.cuda(), kc_dev, vc_dev, tables.cuda(), lens.cuda(), 0.088,
                           max_context_len=int(lens.max()), partition_tokens=0)
    torch.cuda.synchronize()
    ref = oracle.decode(q, kc, vc, tables, lens, 0.088)
    assert_close(out, ref, torch.bfloat16, "manager-driven decode")
    assert pa.device_errors() == 0
