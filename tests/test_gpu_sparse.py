"""GPU parity of the block-sparse calls (sala_block_compress / sala_block_topk /
sala_sparse_prefill / sala_sparse_decode) against the fp64 oracle, through the C ABI.

Compression is checked bit for bit (both sides round the exact mean once).  Selection is checked
with the near-tie rule of tests/parity.py.  Attention is checked on the GPU's own selection (the
oracle re-evaluates the softmax over the blocks the GPU chose), so a legitimate near-tie swap does
not move the output comparison."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sala():
    from hybrid_sparse_linear_b200 import sala as s
    return s


def _f64(t):
    return oracle.from_tensor(t)


def _pipeline(sala, layer, kind, topk, n_init, n_local):
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    kbar = sala.block_compress(k)
    idx = sala.block_topk(q, kbar, topk, n_init, n_local)
    o = sala.sparse_prefill(q, k, v, idx)
    sala.check_status()
    q64, k64, v64 = _f64(layer.q), _f64(layer.k), _f64(layer.v)
    kbar_ref = oracle.block_compress(k64, 64, round_to_bf16=(kind == "bf16"))
    if kind == "f32":
        kbar_ref = kbar_ref.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    idx_ref, kth = oracle.block_select(q64, kbar_ref, 64, topk, n_init, n_local)
    ndiff = check_selection(idx.cpu().numpy(), idx_ref, q64, kbar_ref, kth, topk, n_init, n_local)
    o_ref = oracle.sparse_attention(q64, k64, v64, idx.cpu().numpy(), 64)
    assert_close(_f64(o), o_ref, kind, "o")
    return ndiff


def test_tiny_fp32_pipeline(sala):
    from hybrid_sparse_linear_b200 import synth
    w = synth.WORKLOADS["tiny_fp32_n512"]
    layer = synth.tiny_sparse_layer(1, w["H"], w["Hkv"], w["N"], w["d"], torch.float32, layer=1)
    _pipeline(sala, layer, "f32", w["topk"], w["n_init"], w["n_local"])


@pytest.mark.parametrize("N,topk,n_local", [(64 * 70 + 17, 8, 2), (64 * 40, 64, 2), (64 * 9, 3, 1),
                                             (100, 4, 2), (64 * 300, 16, 2), (64 * 20 + 5, 0, 2)])
def test_bf16_pipeline_gqa16(sala, N, topk, n_local):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=2, shift_frac=0.05)
    _pipeline(sala, layer, "bf16", topk, 1, n_local)


def test_bf16_d64_pipeline_cuda_core_paths(sala):
    # d = 64 runs the CUDA-core selection and attention kernels in bf16.
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 8, 2, 64 * 30 + 3, 64, torch.bfloat16, layer=9, shift_frac=0.1)
    _pipeline(sala, layer, "bf16", 5, 1, 2)


def test_bf16_selection_batch2_k_below_64(sala):
    # batch 2, k = 17 (lists shorter than their 64-entry capacity), tile of rows crossing N.
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(2, 32, 2, 64 * 41 + 30, 128, torch.bfloat16, layer=10, shift_frac=0.05)
    _pipeline(sala, layer, "bf16", 17, 1, 2)


def test_fp32_d128_pipeline_batch2(sala):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(2, 8, 2, 64 * 12 + 5, 128, torch.float32, layer=3, shift_frac=0.1)
    _pipeline(sala, layer, "f32", 3, 1, 2)


@pytest.mark.parametrize("topk", [64, 23])
def test_bf16_selection_weak_pilot(sala, topk):
    # Alternate rows negated: the tile's summed query nearly cancels, so the pilot seeds are close to
    # random and most candidates clear the floor; the row buffers overflow and are cut many times.
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, 64 * 600 + 40, 128, torch.bfloat16, layer=11, shift_frac=0.05)
    q = layer.q.clone()
    q[:, :, 1::2] = -q[:, :, 1::2]
    kbar = sala.block_compress(layer.k.cuda())
    idx = sala.block_topk(q.cuda(), kbar, topk, 1, 2)
    sala.check_status()
    kbar_ref = oracle.block_compress(_f64(layer.k), 64, round_to_bf16=True)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    idx_ref, kth = oracle.block_select(_f64(q), kbar_ref, 64, topk, 1, 2)
    check_selection(idx.cpu().numpy(), idx_ref, _f64(q), kbar_ref, kth, topk, 1, 2)


def test_shifted_blocks_are_selected(sala):
    # Structural invariant on the GPU output: every shifted block that is a candidate is chosen
    # while no more than top-k shifted blocks are causally available.
    from hybrid_sparse_linear_b200 import synth
    N, topk = 64 * 200, 16
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=4, shift_frac=0.05)
    kbar = sala.block_compress(layer.k.cuda())
    idx = sala.block_topk(layer.q.cuda(), kbar, topk, 1, 2).cpu().numpy()
    for g in range(2):
        shifted = layer.shifted[0][g]
        for r in range(0, N, 61):
            c = r // 64
            avail = [x for x in shifted if 1 <= x <= c - 2]
            if len(avail) <= topk:
                assert set(avail) <= set(idx[0, g, r]), (g, r)


def test_out_of_range_index_is_flagged(sala):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, 256, 128, torch.bfloat16, layer=5)
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    idx = torch.full((1, 2, 256, 3), -1, dtype=torch.int32)
    idx[..., 0] = 0
    idx[0, 0, 5, 1] = 3  # block 3 is in the future of row 5
    o = sala.sparse_prefill(q, k, v, idx.cuda())
    with pytest.raises(sala.SalaError) as ei:
        sala.check_status()
    assert ei.value.code == sala.ERR_BOUNDS
    assert torch.isfinite(o.float()).all()
    sala.check_status()  # the word was cleared


# ---------------------------------------------------------------------------------------------
def _decode_case(sala, T, topk, n_init, n_local, dtype, layer_id, given_idx=False, H=32, Hkv=2,
                 d=128, workspace=None, B=1):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(B, H, Hkv, T, d, dtype, device="cuda", layer=layer_id,
                               shift_frac=0.05, q_rows=1)
    pos = T - 1
    kc, vc = layer.k, layer.v
    kbar = sala.block_compress(kc)
    qd = layer.q[:, :, 0].contiguous()
    slots = n_init + n_local + topk
    idx_out = torch.empty((B, Hkv, slots), dtype=torch.int32, device="cuda")
    q64 = _f64(layer.q)
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    kbar_ref = oracle.block_compress(_f64(layer.k), 64, round_to_bf16=(kind == "bf16"))
    if kind == "f32":
        kbar_ref = kbar_ref.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_f64(kbar)[:, :, :kbar_ref.shape[2]], kbar_ref)
    idx_ref, kth = oracle.block_select(q64, kbar_ref, 64, topk, n_init, n_local, q_pos0=pos)
    idx_in = torch.from_numpy(idx_ref[:, :, 0]).cuda() if given_idx else None
    o = sala.sparse_decode(qd, kc, vc, kbar, pos, topk, n_init, n_local, idx_in=idx_in,
                           idx_out=idx_out, workspace=workspace)
    sala.check_status()
    got = idx_out.cpu().numpy()[:, :, None, :]
    check_selection(got, idx_ref, q64, kbar_ref, kth, topk, n_init, n_local, q_pos0=pos,
                    row_ids=np.array([0]))
    o_ref = oracle.sparse_attention(q64, _f64(layer.k), _f64(layer.v), got, 64, q_pos0=pos)
    assert_close(_f64(o), o_ref[:, :, 0], kind, "decode o")
    return o, idx_out


@pytest.mark.parametrize("T", [64 * 300 + 5, 64 * 300, 64 * 3, 1, 70])
def test_sparse_decode(sala, T):
    _decode_case(sala, T, 16, 1, 2, torch.bfloat16, 6)


@pytest.mark.parametrize("T,topk", [(64 * 700 + 9, 64), (64 * 95, 100)])
def test_sparse_decode_batched(sala, T, topk):
    # B = 3 sequences at one position: every (sequence, KV group) selects and attends on its own;
    # k = 100 (past the one-launch kernel; accepted while every candidate is taken, here 92 of
    # them) takes the four-launch path.
    _decode_case(sala, T, topk, 1, 2, torch.bfloat16, 12, B=3)


def test_sparse_decode_given_idx_fp32(sala):
    _decode_case(sala, 64 * 50 + 7, 8, 1, 2, torch.float32, 7, given_idx=True)


def test_sparse_decode_1m_context(sala):
    """One sparse layer at a 2^20-token cache: 16384 compressed blocks, top-64 + init + 2 local."""
    _decode_case(sala, 1 << 20, 64, 1, 2, torch.bfloat16, 8)


def test_sparse_decode_multi_launch_path(sala):
    """k = 100 (103 slots) is past the one-launch kernel's limits: the four-launch path runs.  With
    at most k candidates every block up to the query's is selected."""
    _decode_case(sala, 64 * 90 + 3, 100, 1, 2, torch.bfloat16, 9)


def test_sparse_decode_fp32_d64_one_head_per_group(sala):
    _decode_case(sala, 64 * 200 + 17, 8, 1, 1, torch.float32, 10, H=2, Hkv=2, d=64)


def test_sparse_decode_top0_forced_blocks_only(sala):
    _decode_case(sala, 64 * 40 + 9, 0, 1, 2, torch.bfloat16, 12)


def test_sparse_decode_workspace_reused_across_calls_and_shapes(sala):
    """One zero-filled workspace serves call after call (the grid barrier's counters come back to
    zero), also when the context length changes between calls."""
    T_big, T_small = 64 * 2000 + 5, 64 * 300 + 5
    need = max(sala.sparse_decode_workspace_bytes(1, 32, 2, T - 1, 64, 1, 2, 128)
               for T in (T_big, T_small))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    first = None
    for T in (T_big, T_small, T_big, T_big):
        o, idx = _decode_case(sala, T, 64, 1, 2, torch.bfloat16, 13, workspace=ws)
        torch.cuda.synchronize()
        word = int(ws[:4].view(torch.int32)[0].item())
        assert word & 0xFFFF == 0, f"barrier count not restored: {word:#x}"  # low half: arrivals
        if T == T_big:
            if first is None:
                first = (o.clone(), idx.clone())
            else:
                assert torch.equal(o, first[0]) and torch.equal(idx, first[1])


def test_sparse_decode_bf16_d64_four_heads_per_group(sala):
    # bf16 d = 64 with G = 4: the prefetching one-launch kernel with padding heads in its tiles
    _decode_case(sala, 64 * 900 + 33, 32, 1, 2, torch.bfloat16, 14, H=8, Hkv=2, d=64)


def test_sparse_decode_bf16_given_idx(sala):
    # a given selection: the one-launch kernel attends slots j, j + cpg, ... of the list
    _decode_case(sala, 64 * 500 + 7, 64, 1, 2, torch.bfloat16, 15, given_idx=True)


def test_sparse_decode_clustered_winners_take_the_exact_fallback(sala):
    """The prefetching kernel ranks each CTA's best 8 keys among the group's published ones; when a
    CTA holds more than 8 winners it must fall back to an exact selection over all keys.  The
    candidates are dealt to the group's CTAs in 4-block chunks round robin (74 CTAs per group on a
    148-SM B200 with 2 groups), so planting the 80 best blocks in chunks 0, 74, 148, ... puts all of
    them in one CTA.  Selection and output are checked against the oracle on the planted k-bar."""
    from hybrid_sparse_linear_b200 import synth
    T, topk, n_init, n_local, H, Hkv, d = 1 << 20, 64, 1, 2, 32, 2, 128
    layer = synth.sparse_layer(1, H, Hkv, T, d, torch.bfloat16, device="cuda", layer=17,
                               shift_frac=0.02, q_rows=1)
    kbar = sala.block_compress(layer.k)
    q64, k64 = _f64(layer.q), _f64(layer.k)
    qbar = q64[0].reshape(Hkv, H // Hkv, d).sum(axis=1)                    # [Hkv, d]
    # the planted k-bar starts from the oracle's compression (the GPU's must equal it bitwise)
    kb = oracle.block_compress(k64, 64, round_to_bf16=True)
    np.testing.assert_array_equal(_f64(kbar)[:, :, :kb.shape[2]], kb)
    planted = []
    for t in range(20):
        for r in range(4):
            cand = 74 * 4 * t + r
            blk = n_init + cand
            planted.append(blk)
            i = len(planted)
            for g in range(Hkv):
                kb[0, g, blk] += (20000.0 + 97.0 * i) * qbar[g] / float(qbar[g] @ qbar[g])
    kbar_p = torch.from_numpy(kb).to(torch.bfloat16)
    kb_ref = _f64(kbar_p)
    kbar_p = kbar_p.cuda()
    slots = n_init + n_local + topk
    idx_out = torch.empty((1, Hkv, slots), dtype=torch.int32, device="cuda")
    qd = layer.q[:, :, 0].contiguous()
    o = sala.sparse_decode(qd, layer.k, layer.v, kbar_p, T - 1, topk, n_init, n_local,
                           idx_out=idx_out)
    sala.check_status()
    idx_ref, kth = oracle.block_select(q64, kb_ref, 64, topk, n_init, n_local, q_pos0=T - 1)
    got = idx_out.cpu().numpy()[:, :, None, :]
    check_selection(got, idx_ref, q64, kb_ref, kth, topk, n_init, n_local, q_pos0=T - 1,
                    row_ids=np.array([0]))
    assert set(got[0, 0, 0, n_init:n_init + topk]) <= set(planted)
    o_ref = oracle.sparse_attention(q64, k64, _f64(layer.v), got, 64, q_pos0=T - 1)
    assert_close(_f64(o), o_ref[:, :, 0], "bf16", "decode o")


@pytest.mark.parametrize("graph", [False, True])
def test_hybrid_decode_chain_programmatic_dependents(sala, graph):
    """One token through linear, linear, sparse, linear, sparse layers, every call launched as a
    programmatic dependent of the one before (the linear ones read their state early, the sparse
    ones their share of k-bar); eagerly and replayed from a CUDA graph.  Every layer's output
    against the oracle (the sparse ones through the selection check)."""
    from hybrid_sparse_linear_b200 import synth
    H, Hkv, d, topk, n_init, n_local = 32, 2, 128, 64, 1, 2
    kinds = ["lin", "lin", "sparse", "lin", "sparse"]
    gen = torch.Generator().manual_seed(91)
    lam = synth.decays(H)
    lam_d = lam.cuda()
    layers = []
    for li, kind in enumerate(kinds):
        if kind == "lin":
            S0 = torch.randn((1, H, d, d), generator=gen) / d
            qkv = [(torch.randn((1, H, d), generator=gen) / 4).to(torch.bfloat16) for _ in range(3)]
            layers.append(("lin", S0, [x.cuda() for x in qkv], qkv, S0.clone().cuda()))
        else:
            T = 64 * (1500 + 700 * li) + 11
            sl = synth.sparse_layer(1, H, Hkv, T, d, torch.bfloat16, device="cuda", layer=30 + li,
                                    q_rows=1)
            kbar = sala.block_compress(sl.k)
            ws = torch.zeros(sala.sparse_decode_workspace_bytes(1, H, Hkv, T - 1, topk, n_init,
                                                                n_local, d), dtype=torch.uint8,
                             device="cuda")
            idx = torch.empty((1, Hkv, n_init + n_local + topk), dtype=torch.int32, device="cuda")
            layers.append(("sparse", T, sl, kbar, ws, idx))
    outs = [torch.empty((1, H, d), dtype=torch.bfloat16, device="cuda") for _ in kinds]
    stream = torch.cuda.Stream()

    def run():
        for li, L in enumerate(layers):
            if L[0] == "lin":
                q, k, v = L[2]
                sala.linear_decode(q, k, v, lam_d, L[4], o=outs[li], stream=stream, pdl=True)
            else:
                _, T, sl, kbar, ws, idx = L
                sala.sparse_decode(sl.q[:, :, 0].contiguous(), sl.k, sl.v, kbar, T - 1, topk,
                                   n_init, n_local, idx_out=idx, o=outs[li], workspace=ws,
                                   stream=stream, pdl=True)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        if graph:
            G = torch.cuda.CUDAGraph()
            with torch.cuda.graph(G, stream=stream):
                run()
            for L in layers:  # capture ran nothing; start from the initial states anyway
                if L[0] == "lin":
                    L[4].copy_(L[1])
            G.replay()
        else:
            run()
    torch.cuda.synchronize()
    sala.check_status(stream)
    for li, L in enumerate(layers):
        if L[0] == "lin":
            q, k, v = (_f64(x) for x in L[3])
            o_ref, _ = oracle.linear_decode(q, k, v, _f64(lam), _f64(L[1]))
            assert_close(_f64(outs[li]), o_ref, "bf16", f"layer {li} (linear)")
        else:
            _, T, sl, kbar, ws, idx = L
            q64 = _f64(sl.q)
            kb_ref = oracle.block_compress(_f64(sl.k), 64)
            np.testing.assert_array_equal(_f64(kbar), kb_ref)
            idx_ref, kth = oracle.block_select(q64, kb_ref, 64, topk, n_init, n_local, q_pos0=T - 1)
            got = idx.cpu().numpy()[:, :, None, :]
            check_selection(got, idx_ref, q64, kb_ref, kth, topk, n_init, n_local, q_pos0=T - 1,
                            row_ids=np.array([0]))
            o_ref = oracle.sparse_attention(q64, _f64(sl.k), _f64(sl.v), got, 64, q_pos0=T - 1)
            assert_close(_f64(outs[li]), o_ref[:, :, 0], "bf16", f"layer {li} (sparse)")


def test_sparse_decode_run_twice_bitwise(sala):
    # the same call twice on fresh workspaces gives the same bits (selection and output)
    from hybrid_sparse_linear_b200 import synth
    T = 1 << 19
    sl = synth.sparse_layer(1, 32, 2, T, 128, torch.bfloat16, device="cuda", layer=18, q_rows=1)
    kbar = sala.block_compress(sl.k)
    res = []
    for _ in range(2):
        idx = torch.empty((1, 2, 67), dtype=torch.int32, device="cuda")
        o = sala.sparse_decode(sl.q[:, :, 0].contiguous(), sl.k, sl.v, kbar, T - 1, 64, 1, 2,
                               idx_out=idx)
        sala.check_status()
        res.append((o, idx))
    assert torch.equal(res[0][1], res[1][1]) and torch.equal(res[0][0], res[1][0])


# ---------------------------------------------------------------------------------------------
# Paged KV cache, one position per sequence (sala_sparse_decode_paged)

def _paged_batch(sala, lengths, H=32, Hkv=2, d=128, seed=0, layer0=20):
    """Each sequence drawn dense at its own length, its blocks scattered over a shuffled page
    pool (with unused pages in between).  Returns the paged tensors and the dense originals."""
    from hybrid_sparse_linear_b200 import synth
    B = len(lengths)
    layers = [synth.sparse_layer(1, H, Hkv, n, d, torch.bfloat16, "cpu", layer=layer0 + b,
                                 shift_frac=0.05, q_rows=1) for b, n in enumerate(lengths)]
    nblk = [(n + 63) // 64 for n in lengths]
    max_pages = max(nblk)
    n_pages = sum(nblk) + 7
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    k_pages = torch.zeros((n_pages, Hkv, 64, d), dtype=torch.bfloat16)
    v_pages = torch.zeros_like(k_pages)
    nxt = 0
    for b, (sl, n) in enumerate(zip(layers, lengths)):
        for j in range(nblk[b]):
            p = int(perm[nxt]); nxt += 1
            table[b, j] = p
            rows = min(64, n - 64 * j)
            k_pages[p, :, :rows] = sl.k[0, :, 64 * j:64 * j + rows]
            v_pages[p, :, :rows] = sl.v[0, :, 64 * j:64 * j + rows]
    nb_cap = max(n // 64 for n in lengths)
    kbar = torch.zeros((B, Hkv, max(nb_cap, 1), d), dtype=torch.bfloat16, device="cuda")
    for b, sl in enumerate(layers):
        nb = lengths[b] // 64
        if nb:
            kbar[b, :, :nb] = sala.block_compress(sl.k.cuda())[0, :, :nb]
    q = torch.stack([sl.q[0, :, 0] for sl in layers]).contiguous()
    pos = torch.tensor([n - 1 for n in lengths], dtype=torch.int32)
    return (q.cuda(), k_pages.cuda(), v_pages.cuda(), torch.from_numpy(table).cuda(), kbar,
            pos.cuda(), layers)


def test_sparse_decode_paged_per_sequence_positions(sala):
    lengths = [64 * 300 + 5, 64 * 40, 64 * 3 + 1, 64 * 128]
    topk, n_init, n_local = 64, 1, 2
    q, kp, vp, table, kbar, pos, layers = _paged_batch(sala, lengths)
    B, Hkv = len(lengths), kp.shape[1]
    idx_out = torch.empty((B, Hkv, n_init + n_local + topk), dtype=torch.int32, device="cuda")
    o = sala.sparse_decode_paged(q, kp, vp, table, kbar, pos, max(lengths) - 1, topk, n_init,
                                 n_local, idx_out=idx_out)
    sala.check_status()
    got = idx_out.cpu().numpy()
    for b, (sl, n) in enumerate(zip(layers, lengths)):
        p = n - 1
        q64, k64, v64 = _f64(sl.q), _f64(sl.k), _f64(sl.v)
        kbar_ref = oracle.block_compress(k64, 64, round_to_bf16=True) if n >= 64 else \
            np.zeros((1, Hkv, 0, q64.shape[-1]))
        idx_ref, kth = oracle.block_select(q64, kbar_ref, 64, topk, n_init, n_local, q_pos0=p)
        gb = got[b:b + 1, :, None, :]
        check_selection(gb, idx_ref, q64, kbar_ref, kth, topk, n_init, n_local, q_pos0=p,
                        row_ids=np.array([0]))
        o_ref = oracle.sparse_attention(q64, k64, v64, gb, 64, q_pos0=p)
        assert_close(_f64(o[b:b + 1]), o_ref[:, :, 0], "bf16", f"paged decode sequence {b}")


def test_sparse_decode_paged_bad_page_is_flagged(sala):
    lengths = [64 * 50 + 3, 64 * 20]
    q, kp, vp, table, kbar, pos, _ = _paged_batch(sala, lengths, seed=1)
    table[0, 0] = kp.shape[0] + 5          # block 0 (always attended) names no page
    sala.sparse_decode_paged(q, kp, vp, table, kbar, pos, max(lengths) - 1, 16, 1, 2)
    with pytest.raises(sala.SalaError) as e:
        sala.check_status()
    assert e.value.code == sala.ERR_BOUNDS
    # the context stays usable: a good call afterwards succeeds
    table[0, 0] = 0 if int(table[1, 0]) != 0 else 1
    sala.sparse_decode_paged(q, kp, vp, table, kbar, pos, max(lengths) - 1, 16, 1, 2)
    sala.check_status()


# ---------------------------------------------------------------------------------------------
# Query-block-granular selection (sala_block_topk_qblock)

@pytest.mark.parametrize("N,topk,dtype,d,H,Hkv", [
    (64 * 200 + 7, 64, torch.bfloat16, 128, 32, 2),   # 16 heads per group, partial last block
    (64 * 30 + 5, 8, torch.float32, 64, 8, 2),        # fp32, d 64
    (64 * 4500 + 9, 64, torch.bfloat16, 128, 2, 1),   # > 4032 candidates: winners carried over chunks
])
def test_qblock_selection(sala, N, topk, dtype, d, H, Hkv):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, H, Hkv, N, d, dtype, layer=13, shift_frac=0.05)
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    q, k = layer.q.cuda(), layer.k.cuda()
    kbar = sala.block_compress(k)
    idx = sala.block_topk_qblock(q, kbar, topk, 1, 2)
    sala.check_status()
    kbar_ref = oracle.block_compress(_f64(layer.k), 64, round_to_bf16=(kind == "bf16"))
    if kind == "f32":
        kbar_ref = kbar_ref.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    q64 = _f64(layer.q)
    ref, kth = oracle.block_select_qblock(q64, kbar_ref, 64, topk, 1, 2)
    got = idx.cpu().numpy()
    for r0 in range(0, N, 64):   # one row per query block on the GPU too
        assert (got[:, :, r0:r0 + 64] == got[:, :, r0:r0 + 1]).all(), r0
    check_selection(got, ref, oracle.qblock_sum(q64, 64), kbar_ref, kth, topk, 1, 2)


def test_qblock_pipeline(sala):
    # sparse prefill over query-block selections (every unit of 16 tokens shares one selection)
    from hybrid_sparse_linear_b200 import synth
    N, topk = 64 * 90 + 21, 32
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=14, shift_frac=0.05)
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    kbar = sala.block_compress(k)
    idx = sala.block_topk_qblock(q, kbar, topk, 1, 2)
    o = sala.sparse_prefill(q, k, v, idx)
    sala.check_status()
    q64, k64, v64 = _f64(layer.q), _f64(layer.k), _f64(layer.v)
    kbar_ref = oracle.block_compress(k64, 64, round_to_bf16=True)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    ref, kth = oracle.block_select_qblock(q64, kbar_ref, 64, topk, 1, 2)
    got = idx.cpu().numpy()
    check_selection(got, ref, oracle.qblock_sum(q64, 64), kbar_ref, kth, topk, 1, 2)
    assert_close(_f64(o), oracle.sparse_attention(q64, k64, v64, got, 64), "bf16", "o")


# ---------------------------------------------------------------------------------------------
# Query-block selection scored by softmax-probability group aggregation

def _check_softmax_selection(got, ref, kth, q64, kbar_ref, topk, n_init, n_local, rel=1e-3):
    """Rows may differ only by near-ties: every block in the symmetric difference scores within
    rel of the oracle's k-th score (scores from the oracle's fp64 helper)."""
    B, Hkv, N, _ = got.shape
    for b in range(B):
        for g in range(Hkv):
            for r0 in range(0, N, 64):
                a, e = got[b, g, r0], ref[b, g, r0]
                assert (got[b, g, r0:r0 + 64] == a).all(), (b, g, r0)
                if (a == e).all():
                    continue
                c = r0 // 64
                ids, sc = oracle.qblock_softmax_scores(q64, kbar_ref, 64, b, g, c, n_init, n_local)
                score = dict(zip(ids.tolist(), sc.tolist()))
                sa, se = {x for x in a if x >= 0}, {x for x in e if x >= 0}
                assert len(sa) == len(se), (b, g, c)
                k = kth[b, g, r0]
                for x in sa ^ se:
                    assert x in score, f"block {x} is not a candidate of query block {c}"
                    assert abs(score[x] - k) <= rel * max(abs(score[x]), abs(k)), \
                        f"query block {c}: block {x} scores {score[x]}, k-th {k}"


@pytest.mark.parametrize("N,topk,dtype,d,H,Hkv", [
    (64 * 200 + 7, 64, torch.bfloat16, 128, 32, 2),   # 16 heads per group, partial last block
    (64 * 30 + 5, 8, torch.float32, 64, 8, 2),        # fp32, d 64
    (64 * 4500 + 9, 64, torch.bfloat16, 128, 4, 2),   # > 4032 candidates: winners carried over chunks
])
def test_qblock_softmax_selection(sala, N, topk, dtype, d, H, Hkv):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, H, Hkv, N, d, dtype, layer=15, shift_frac=0.05)
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    q, k = layer.q.cuda(), layer.k.cuda()
    kbar = sala.block_compress(k)
    idx = sala.block_topk_qblock_softmax(q, kbar, topk, 1, 2)
    sala.check_status()
    kbar_ref = oracle.block_compress(_f64(layer.k), 64, round_to_bf16=(kind == "bf16"))
    if kind == "f32":
        kbar_ref = kbar_ref.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    q64 = _f64(layer.q)
    ref, kth = oracle.block_select_qblock_softmax(q64, kbar_ref, 64, topk, 1, 2)
    _check_softmax_selection(idx.cpu().numpy(), ref, kth, q64, kbar_ref, topk, 1, 2)


def test_qblock_softmax_pipeline(sala):
    from hybrid_sparse_linear_b200 import synth
    N, topk = 64 * 90 + 21, 32
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=16, shift_frac=0.05)
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    kbar = sala.block_compress(k)
    idx = sala.block_topk_qblock_softmax(q, kbar, topk, 1, 2)
    o = sala.sparse_prefill(q, k, v, idx)
    sala.check_status()
    q64, k64, v64 = _f64(layer.q), _f64(layer.k), _f64(layer.v)
    kbar_ref = oracle.block_compress(k64, 64, round_to_bf16=True)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    ref, kth = oracle.block_select_qblock_softmax(q64, kbar_ref, 64, topk, 1, 2)
    got = idx.cpu().numpy()
    _check_softmax_selection(got, ref, kth, q64, kbar_ref, topk, 1, 2)
    assert_close(_f64(o), oracle.sparse_attention(q64, k64, v64, got, 64), "bf16", "o")
