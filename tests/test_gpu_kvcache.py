"""GPU parity of the FP8 (E4M3) KV cache against the oracle: the append
kernel's codes and scales bit for bit (the per-token rule on every
(token, KV head) vector), and decode attention over the paged cache within
|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) of the oracle's fp64 attention,
over context lengths around the 16- and 128-position tiles and the
512-position chunks, GQA groups of 1 to 16 query heads, head sizes 64 and
128, and block tables with missing entries.  Every attention case runs on
both kernels: the warp-level one ("mma") and the tensor-memory one ("tc",
for the shapes it takes; the others fall back to "mma", which the test
checks)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from helpers import assert_gemm_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


@pytest.fixture(params=["mma", "tc"])
def kernel(request, ptpc, monkeypatch):
    monkeypatch.setenv("PTPC_FORCE_ATTN_KERNEL", request.param)
    ptpc.reload_tuning_overrides()
    yield request.param
    monkeypatch.delenv("PTPC_FORCE_ATTN_KERNEL")
    ptpc.reload_tuning_overrides()


def expect_kernel(ptpc, kernel, Hq, Hkv, D, bs):
    tc_shape = D == 128 and Hq // Hkv <= 16 and bs % 8 == 0
    assert ptpc.decode_attention_kernel(Hq, Hkv, D, bs) == ("tc" if kernel == "tc" and tc_shape else "mma")


def run_attention(ptpc, q, kc, vc, ksc, vsc, tables, lens, max_ctx, scale):
    """decode_attention through an explicit zeroed workspace whose device
    status word must still be clear afterwards."""
    B, Hq, D = q.shape
    ws = ptpc.Workspace(ptpc.lib.ptpc_decode_attention_workspace_size(B, Hq, D, max_ctx), "cuda")
    out = ptpc.decode_attention(to_dev_bf16(q), kc, vc, ksc, vsc, torch.from_numpy(tables).cuda(),
                                torch.tensor(lens, dtype=torch.int32, device="cuda"), max_ctx, scale, ws=ws)
    assert ptpc.device_status(ws) == 0
    return from_dev_bf16(out)


def make_kv(T, H, D, seed, ramp=0.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((T, H, D)).astype(np.float32)
    x *= rng.lognormal(0.0, 1.0, size=(T, H, 1)).astype(np.float32)
    x[:, :, rng.choice(D, 2, replace=False)] *= 20.0          # a few outlier channels per head
    if ramp:
        x *= (1.0 + ramp * np.arange(T, dtype=np.float32))[:, None, None]
    return synthetic.to_bf16_bits(x)


def build_cache(ptpc, lens, Hkv, D, bs, seed, holes=False, ramp=0.0):
    """Random block tables, K/V appended through the library; returns device
    caches and the oracle's copies."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B = len(lens)
    max_blocks = max(1, max((l + bs - 1) // bs for l in lens))
    nb = B * max_blocks + 3
    perm = rng.permutation(nb)
    tables = np.full((B, max_blocks), -1, np.int32)
    k = 0
    for b, l in enumerate(lens):
        n = (l + bs - 1) // bs
        tables[b, :n] = perm[k:k + n]
        k += n
    slots = []
    for b, l in enumerate(lens):
        for pos in range(l):
            slots.append(tables[b, pos // bs] * bs + pos % bs)
    T = len(slots)
    K = make_kv(max(T, 1), Hkv, D, seed + 1, ramp)[:T]
    V = make_kv(max(T, 1), Hkv, D, seed + 2, ramp)[:T]
    kc = torch.zeros((nb, bs, Hkv, D), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    ksc = torch.zeros((nb, bs, Hkv), dtype=torch.float32, device="cuda")
    vsc = torch.zeros_like(ksc)
    if T:
        ptpc.kv_cache_append(to_dev_bf16(K), to_dev_bf16(V), torch.tensor(slots, dtype=torch.int64, device="cuda"),
                             kc, vc, ksc, vsc)
    rk = np.zeros((nb, bs, Hkv, D), np.uint8); rv = np.zeros_like(rk)
    rks = np.zeros((nb, bs, Hkv), np.float32); rvs = np.zeros_like(rks)
    if T:
        qk, sk = oracle.kv_quantize(K)
        qv, sv = oracle.kv_quantize(V)
        oracle.kv_cache_write(rk, rks, qk, sk, slots, bs)
        oracle.kv_cache_write(rv, rvs, qv, sv, slots, bs)
    if holes and max_blocks > 2:
        tables[0, 1] = -1          # a missing block: its positions are left out on both sides
    return (kc, vc, ksc, vsc, tables), (rk, rv, rks, rvs)


def test_append_bit_exact(ptpc):
    T, H, D, bs, nb = 300, 8, 128, 16, 32
    K = make_kv(T, H, D, 1)
    V = make_kv(T, H, D, 2)
    K[3] = 0x8000                      # an all -0 token: scale 1, codes 0
    rng = np.random.Generator(np.random.PCG64(3))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[5] = -1                      # skipped
    slots[6] = nb * bs + 7             # past the cache: skipped
    kc = torch.full((nb, bs, H, D), 0xAB, dtype=torch.uint8, device="cuda")
    vc = kc.clone()
    ksc = torch.full((nb, bs, H), -7.0, device="cuda")
    vsc = ksc.clone()
    ptpc.kv_cache_append(to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(slots).cuda(), kc, vc, ksc, vsc)
    rk = np.full((nb, bs, H, D), 0xAB, np.uint8); rv = rk.copy()
    rks = np.full((nb, bs, H), -7.0, np.float32); rvs = rks.copy()
    keep = [t for t in range(T) if 0 <= slots[t] < nb * bs]
    qk, sk = oracle.kv_quantize(K[keep])
    qv, sv = oracle.kv_quantize(V[keep])
    oracle.kv_cache_write(rk, rks, qk, sk, slots[keep], bs)
    oracle.kv_cache_write(rv, rvs, qv, sv, slots[keep], bs)
    assert np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(vc.cpu().numpy(), rv)
    assert np.array_equal(ksc.cpu().numpy().view(np.uint32), rks.view(np.uint32))
    assert np.array_equal(vsc.cpu().numpy().view(np.uint32), rvs.view(np.uint32))


@pytest.mark.parametrize("lens,Hq,Hkv,D,bs", [
    ([1, 15, 16, 17, 100], 8, 1, 128, 16),
    ([511, 512, 513, 1030], 64, 8, 128, 16),
    ([33, 700], 16, 16, 128, 32),
    ([257, 1500], 32, 2, 64, 16),
    ([0, 5, 2049], 28, 4, 128, 16),
    ([1, 127, 128, 129, 255, 256, 1000, 2047], 24, 3, 128, 8),
    ([130, 641], 12, 12, 128, 48),
    ([1, 300, 1000, 4097], 32, 2, 128, 16),      # groups of 16: two CTAs a KV head
    ([77, 2100], 24, 2, 128, 8),                 # groups of 12: 8 + 4 heads
])
def test_decode_attention(ptpc, kernel, lens, Hq, Hkv, D, bs):
    _attention_case(ptpc, kernel, lens, Hq, Hkv, D, bs)


@pytest.mark.parametrize("chunk", ["1024", "2048", "4096"])
@pytest.mark.parametrize("lens,Hq,Hkv,D,bs", [
    ([511, 512, 513, 1030, 2047, 2048, 2049, 4100, 8200], 64, 8, 128, 16),
    ([257, 1500, 3000], 32, 2, 64, 24),
    ([0, 5, 2049], 28, 4, 128, 16),
])
def test_decode_attention_chunk_sizes(ptpc, monkeypatch, kernel, chunk, lens, Hq, Hkv, D, bs):
    """The larger context chunks a CTA can take (chosen by the launch for
    long contexts on many sequences; 4096 only on the tensor-memory kernel,
    the warp-level one takes 2048), forced on small cases; a block size that
    is not a power of two exercises the exact quotient."""
    monkeypatch.setenv("PTPC_FORCE_ATTN_CHUNK", chunk)
    ptpc.reload_tuning_overrides()
    try:
        _attention_case(ptpc, kernel, lens, Hq, Hkv, D, bs)
    finally:
        monkeypatch.delenv("PTPC_FORCE_ATTN_CHUNK")
        ptpc.reload_tuning_overrides()


def _attention_case(ptpc, kernel, lens, Hq, Hkv, D, bs, ramp=0.0):
    expect_kernel(ptpc, kernel, Hq, Hkv, D, bs)
    dev, ref = build_cache(ptpc, lens, Hkv, D, bs, seed=sum(lens) + Hq, holes=True, ramp=ramp)
    kc, vc, ksc, vsc, tables = dev
    rk, rv, rks, rvs = ref
    assert np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(vsc.cpu().numpy(), rvs)
    B = len(lens)
    rng = np.random.Generator(np.random.PCG64(11))
    q = synthetic.to_bf16_bits(rng.standard_normal((B, Hq, D)).astype(np.float32) * 2.0)
    scale = 1.0 / math.sqrt(D)
    max_ctx = max(lens)
    # the oracle over the same table (missing entries: positions left out)
    got = run_attention(ptpc, q, kc, vc, ksc, vsc, tables, lens, max_ctx, scale)
    for b in range(B):
        L = lens[b]
        pos = [p for p in range(L) if tables[b, p // bs] >= 0]
        if not pos:
            assert not got[b].any() or np.all((got[b] & 0x7FFF) == 0)
            continue
        bt = np.array([[tables[b, p // bs] for p in pos]])
        offs = [p % bs for p in pos]
        # gather the positions into a one-position-per-block table for the reference
        ck = rk[bt[0], offs][None].transpose(1, 0, 2, 3)     # [n, 1, Hkv, D]
        cv = rv[bt[0], offs][None].transpose(1, 0, 2, 3)
        cks = rks[bt[0], offs][:, None, :]
        cvs = rvs[bt[0], offs][:, None, :]
        r = oracle.decode_attention_reference(q[b:b + 1], ck, cks, cv, cvs, np.arange(len(pos))[None],
                                              [len(pos)], 1, scale)
        assert_gemm_close(got[b:b + 1], r, f"attention b={b} L={L} Hq={Hq} Hkv={Hkv} D={D}")


def test_decode_attention_growing_scores(ptpc, kernel):
    """Keys and values whose size grows along the context (x 1 + t / 40):
    the running maximum of every head and the largest value scale move many
    times within a chunk, so the kernels rescale their accumulators often."""
    _attention_case(ptpc, kernel, [300, 1000, 2100], 16, 2, 128, 16, ramp=1.0 / 40)


def test_decode_attention_70b_shape(ptpc, kernel):
    """Llama-3.1-70B attention at decode: 64 query heads on 8 KV heads, D =
    128, 16-position blocks; a batch of mixed context lengths."""
    expect_kernel(ptpc, kernel, 64, 8, 128, 16)
    lens = [4096, 1, 3000, 2048, 777, 4095]
    dev, ref = build_cache(ptpc, lens, 8, 128, 16, seed=70)
    kc, vc, ksc, vsc, tables = dev
    rk, rv, rks, rvs = ref
    rng = np.random.Generator(np.random.PCG64(12))
    q = synthetic.to_bf16_bits(rng.standard_normal((len(lens), 64, 128)).astype(np.float32))
    got = run_attention(ptpc, q, kc, vc, ksc, vsc, tables, lens, 4096, 1 / math.sqrt(128))
    r = oracle.decode_attention_reference(q, rk, rks, rv, rvs, tables, lens, 16, 1 / math.sqrt(128))
    assert_gemm_close(got, r, "70B decode attention")


@pytest.mark.parametrize("q_scale", [1e-39, 1e-20, 1e20, 3e37])
def test_decode_attention_query_range(ptpc, kernel, q_scale):
    """Query vectors far from unit size (bf16 subnormals up to near the bf16
    maximum, times a softmax scale that keeps the scores finite): the
    power-of-two scale of the query's two E4M3 terms keeps them in range."""
    lens, Hq, Hkv, D, bs = [37, 130], 16, 2, 128, 16
    dev, ref = build_cache(ptpc, lens, Hkv, D, bs, seed=5)
    kc, vc, ksc, vsc, tables = dev
    rk, rv, rks, rvs = ref
    rng = np.random.Generator(np.random.PCG64(21))
    qf = rng.standard_normal((len(lens), Hq, D)).astype(np.float32) * np.float32(q_scale)
    q = synthetic.to_bf16_bits(qf)
    scale = float(min(1.0, 1.0 / (q_scale * math.sqrt(D))))
    got = run_attention(ptpc, q, kc, vc, ksc, vsc, tables, lens, max(lens), scale)
    r = oracle.decode_attention_reference(q, rk, rks, rv, rvs, tables, lens, bs, scale)
    assert_gemm_close(got, r, f"attention, |q| ~ {q_scale}")
