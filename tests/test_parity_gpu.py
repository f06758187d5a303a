"""CUDA path vs. the fp64 oracle on identical seeded inputs (element by element).

Tolerance on the bf16 outputs, per call: max |err| <= 2e-2 and mean |err| <= 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
from gpu_helpers import (MAX_ABS_TOL, MEAN_ABS_TOL, assert_parity, device_qkv, needs_gpu,
                         run_cuda)

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("c", si.ENCODER_WORKLOADS, ids=lambda c: c.name)
def test_encoder_workloads_every_call(c):
    """Every seeded layer call of the four encoder workloads."""
    for call in range(c.calls):
        bits = c.qkv(call)
        want = oracle.attention_packed_bf16(bits, c.scale)
        got = run_cuda(bits, c.scale)
        assert_parity(got, want, f"{c.name} call {call}")


# Boundaries of 128-row query tiles / 128-key blocks (d=64) and 112-key blocks (d=72).
EDGE_N = [1, 2, 15, 16, 17, 63, 64, 65, 111, 112, 113, 127, 128, 129, 200, 224, 225, 255, 256,
          257, 336, 337, 383, 384, 385, 448, 449, 511, 512, 513, 560, 561, 576, 577]


@pytest.mark.parametrize("d", [64, 72])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_token_counts(N, d):
    """Ragged query tiles and key blocks, single- and two-slot rounds, ring streaming (d=72, N>560)."""
    B, H = 2, 3
    bits = si.packed_qkv(B, N, H, d, seed=70000 + 10 * N + d)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    got = run_cuda(bits, scale)
    assert_parity(got, want, f"B={B} N={N} H={H} d={d}")


# Longer sequences (384 px and 448 px ViT/14 grids and beyond): K/V resident while a
# head's blocks fit the ring (d=64: N <= 768, d=72: N <= 560), streamed per round after.
LONG_N = [578, 640, 641, 729, 730, 768, 769, 1025, 2049]


@pytest.mark.parametrize("d", [64, 72])
@pytest.mark.parametrize("N", LONG_N)
def test_long_sequences(N, d):
    B, H = 1, 2
    bits = si.packed_qkv(B, N, H, d, seed=90000 + 10 * N + d)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    got = run_cuda(bits, scale)
    assert_parity(got, want, f"B={B} N={N} H={H} d={d}")


def test_longest_sequence_sampled_rows():
    """N = 16384 (the accepted maximum), one head per image, rows sampled across all
    128 query tiles, against the oracle computed row by row."""
    B, N, H, d = 2, 16384, 1, 64
    bits = si.packed_qkv(B, N, H, d, seed=91234)
    scale = 0.125
    import vit_self_attention_b200 as vab
    out = vab.attention(device_qkv(bits), scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    rows = [(b, 0, n) for b in range(B) for n in (0, 1, 127, 128, 8191, 8192, N - 2, N - 1)]
    rows += [(int(rng.integers(0, B)), 0, int(rng.integers(0, N))) for _ in range(120)]
    want = oracle.attention_rows_packed_bf16(bits, scale, rows)
    idx = torch.tensor(rows, dtype=torch.long, device="cuda")
    got = out[idx[:, 0], idx[:, 2], idx[:, 1]].float().cpu().numpy().astype(np.float64)
    assert_parity(got, want, "B=2 N=16384 H=1 sampled rows")


@pytest.mark.parametrize("B,H,N,d", [(8, 4, 577, 64), (4, 5, 1025, 64), (6, 5, 600, 72),
                                     (160, 1, 197, 64), (10, 16, 257, 64), (12, 13, 577, 64),
                                     (75, 2, 577, 72), (1, 1, 577, 64), (148, 1, 129, 72),
                                     (300, 1, 50, 64), (10, 16, 1025, 64), (149, 1, 577, 64),
                                     (297, 1, 300, 64), (157, 1, 600, 72), (10, 16, 700, 64),
                                     (10, 16, 500, 72), (10, 16, 512, 64), (10, 16, 448, 72)])
def test_schedules(B, H, N, d):
    """Whole-head work units (B*H >= #SMs), per-round units (fewer heads, more tiles than
    SMs; K/V streamed when a head's blocks do not fit the ring), single-tile units (all
    tiles fit on the SMs), persistent multi-unit CTAs, and stream mode (whole heads with an
    odd tile count: tiles paired across head boundaries, a lone last tile on CTAs with an
    odd tile total, K/V streamed, with and without the long-sequence ring wrap).  The
    shared-memory plans: two Q buffers with a ring of 4 and the output staging (N=512 /
    448: a head's K/V resident), and whole heads of 6 (d=64, N=700) or 5 (d=72, N=500)
    key blocks, resident only in the longer ring without the staging (row stores)."""
    bits = si.packed_qkv(B, N, H, d, seed=90000 + B * 7 + H * 3 + N + d)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    got = run_cuda(bits, scale)
    assert_parity(got, want, f"B={B} N={N} H={H} d={d}")


@pytest.mark.parametrize("sigma", [2.0, 4.0])
@pytest.mark.parametrize("d", [64, 72])
def test_peaked_softmax(sigma, d):
    """Large logits: the running maximum grows across key blocks, exercising the O rescale."""
    B, N, H = 2, 577, 4
    bits = si.packed_qkv(B, N, H, d, seed=int(50000 + sigma * 10 + d), sigma_qk=sigma)
    # Make later keys larger so the row maximum keeps growing block after block.
    x = si.bf16_bits_to_f32(bits).copy()
    ramp = (1.0 + 2.0 * np.arange(N, dtype=np.float32) / N)[None, :, None, None]
    x[:, :, 1] *= ramp
    bits = si.f32_to_bf16_bits(x)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    got = run_cuda(bits, scale)
    assert_parity(got, want, f"sigma={sigma} d={d}")


@pytest.mark.parametrize("d", [64, 72])
@pytest.mark.parametrize("boost", [2.0, 6.0, 40.0])
def test_running_offset_fix_up_positions(d, boost):
    """Keys whose logits jump far above everything before them, placed in later key blocks
    at different 16-key chunks (first, middle and last chunk of a block, and the ragged last
    block): the kernel's weights against the stale running offset fail the chunk check
    there, and the offset is raised with the chunks already stored, the running sum and O
    rescaled.  With boost 40 the jump exceeds the fp32 range of 2^x (an overflow to inf
    that the check must catch).  Every query row is compared with the oracle."""
    B, N, H = 2, 577, 3
    bits = si.packed_qkv(B, N, H, d, seed=int(61000 + boost * 10 + d))
    x = si.bf16_bits_to_f32(bits).copy()
    u = x[:, :1, 0].copy()                     # one direction per image and head
    x[:, :, 0] = 0.25 * x[:, :, 0] + u          # every query leans towards u
    bk = 128 if d == 64 else 112
    spikes = [bk + 5, 2 * bk + 8 * 7, 3 * bk + bk - 3, N - 1]  # blocks 1-3 and the tail
    for rank, j in enumerate(spikes):
        x[:, j, 1] = u[:, 0] * (boost * (rank + 1) / np.sqrt(d))
    bits = si.f32_to_bf16_bits(x)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    got = run_cuda(bits, scale)
    assert_parity(got, want, f"boost={boost} d={d}")


def test_closed_form_inputs_on_gpu():
    """Identical V rows -> O rows equal V; Q = 0 -> O = mean of V (in bf16 precision)."""
    B, N, H, d = 2, 300, 2, 64
    bits = si.packed_qkv(B, N, H, d, seed=4242)
    x = si.bf16_bits_to_f32(bits).copy()
    x[:, :, 2] = x[:, :1, 2]  # every value row equals token 0's
    got = run_cuda(si.f32_to_bf16_bits(x), 0.125)
    want = np.broadcast_to(x[:, :1, 2], (B, N, H, d)).astype(np.float64)
    assert_parity(got, want, "identical V rows", max_tol=1e-2, mean_tol=2e-3)
    x2 = si.bf16_bits_to_f32(bits).copy()
    x2[:, :, 0] = 0.0
    got2 = run_cuda(si.f32_to_bf16_bits(x2), 0.125)
    want2 = np.broadcast_to(x2[:, :, 2].astype(np.float64).mean(axis=1, keepdims=True),
                            (B, N, H, d))
    assert_parity(got2, want2, "Q = 0 -> mean of V")


def test_large_config_every_output():
    """The 336 px ViT-L/14 batch (B=256, N=577, H=16, d=64) in the bench's launch
    configuration (one call over the whole batch: stream mode, one CTA per SM): every
    one of the 151 M outputs against the oracle, with max |err| and mean |err| taken over
    the whole call; also every output inside the per-channel range of its head's value
    rows (O is a convex combination of V rows).  The oracle runs in chunks of whole
    images so that host memory stays bounded."""
    c = si.VIT_L14_336PX_B256
    bits = c.qkv(0)
    qkv = device_qkv(bits)
    import vit_self_attention_b200 as vab
    out = vab.attention(qkv, c.scale)
    torch.cuda.synchronize()
    v = qkv[:, :, 2].float()  # [B, N, H, d]
    lo = v.amin(dim=1, keepdim=True)
    hi = v.amax(dim=1, keepdim=True)
    of = out.float()
    assert torch.isfinite(of).all()
    slack = 1e-2 * (hi - lo) + 1e-3
    assert bool(((of >= lo - slack) & (of <= hi + slack)).all()), "output outside value hull"
    del v, lo, hi, of
    got_all = out.view(torch.int16).cpu().numpy().view(np.uint16)
    worst, total, count = 0.0, 0.0, 0
    step = 32
    for b0 in range(0, c.B, step):
        want = oracle.attention_packed_bf16(bits[b0:b0 + step], c.scale)
        got = si.bf16_bits_to_f32(got_all[b0:b0 + step]).astype(np.float64)
        assert np.all(np.isfinite(got))
        diff = np.abs(got - want)
        worst = max(worst, float(diff.max()))
        total += float(diff.sum())
        count += diff.size
    mean = total / count
    assert count == c.B * c.N * c.H * c.d
    assert worst <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (
        f"B=256 N=577 H=16 d=64, all outputs: max|err| {worst:.3e}, mean|err| {mean:.3e}")


def test_graph_capture_replay():
    """The call can be captured in a CUDA graph and replayed (pointers stay fixed)."""
    import vit_self_attention_b200 as vab
    c = si.VIT_L14_224PX_3VIEWS
    bits = c.qkv(0)
    qkv = device_qkv(bits)
    out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        vab.attention(qkv, c.scale, out=out, stream=s)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        vab.attention(qkv, c.scale, out=out, stream=s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    want = oracle.attention_packed_bf16(bits, c.scale)
    assert_parity(out.float().cpu().numpy().astype(np.float64), want, "graph replay")
    bits2 = c.qkv(1)
    qkv.copy_(device_qkv(bits2))
    g.replay()
    torch.cuda.synchronize()
    want2 = oracle.attention_packed_bf16(bits2, c.scale)
    assert_parity(out.float().cpu().numpy().astype(np.float64), want2, "graph replay, new input")


def test_host_buffer_entry():
    """vla_attn_fwd_host: pinned host input -> device -> kernel -> pinned host output."""
    import vit_self_attention_b200 as vab
    c = si.SIGLIP_SO400M14_224PX_2VIEWS
    bits = c.qkv(5)
    host_in = torch.from_numpy(bits.view(np.int16).copy()).pin_memory()
    host_out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.int16).pin_memory()
    dev_in = torch.empty(bits.shape, dtype=torch.int16, device="cuda")
    dev_out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.int16, device="cuda")
    vab.vla_attn_fwd_host(host_in, host_out, dev_in, dev_out, c.B, c.N, c.H, c.d, c.scale)
    torch.cuda.synchronize()
    got = si.bf16_bits_to_f32(host_out.numpy().view(np.uint16)).astype(np.float64)
    want = oracle.attention_packed_bf16(bits, c.scale)
    assert_parity(got, want, "host-buffer entry")


@pytest.mark.parametrize("full_chunks", [2, 7])
def test_host_buffer_entry_pipelined_chunks(full_chunks):
    """A batch of several chunks (a chunk = the fewest whole images with one head per SM)
    takes the pipelined host path (copy-in and copy-out streams): the host result equals
    the device entry's bytes on the whole batch, on two calls in a row."""
    import vit_self_attention_b200 as vab
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    H, N, d = 16, 197, 64
    chunk = -(-sm // H)
    B = full_chunks * chunk + 3  # full chunks and a ragged one
    bits = si.packed_qkv(B, N, H, d, seed=4242)
    scale = 1.0 / math.sqrt(d)
    host_in = torch.from_numpy(bits.view(np.int16).copy()).pin_memory()
    dev_in = torch.empty(bits.shape, dtype=torch.int16, device="cuda")
    dev_out = torch.empty((B, N, H, d), dtype=torch.int16, device="cuda")
    ref = vab.attention(host_in.cuda().view(torch.bfloat16), scale).view(torch.int16).cpu()
    for _ in range(2):
        host_out = torch.full((B, N, H, d), -1, dtype=torch.int16).pin_memory()
        vab.vla_attn_fwd_host(host_in, host_out, dev_in, dev_out, B, N, H, d, scale)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(host_out, ref)
    rows = [(0, 0, 0), (chunk, 5, 196), (B - 1, 15, 100)]
    got = si.bf16_bits_to_f32(host_out.numpy().view(np.uint16)).astype(np.float64)
    want = oracle.attention_rows_packed_bf16(bits, scale, rows)
    assert_parity(np.stack([got[b, n, h] for b, h, n in rows]), want, "pipelined host entry")


def test_device_status_clean_and_launch_count():
    import vit_self_attention_b200 as vab
    n0 = vab.vla_attn_launch_count()
    run_cuda(si.VIT_B16_112PX_1VIEW.qkv(0), si.VIT_B16_112PX_1VIEW.scale)
    assert vab.vla_attn_launch_count() == n0 + 1
    st, site = vab.vla_attn_last_device_status()
    assert st == 0 and site == 0


def test_rejects_host_and_short_buffers():
    """Pointers that are not device memory, allocations too small for the shape, and an
    output overlapping the input are refused before anything is launched."""
    import vit_self_attention_b200 as vab
    from cuda.bindings import runtime as cudart
    B, N, H, d = 1, 50, 12, 64
    in_bytes = B * N * 3 * H * d * 2
    out = torch.empty(B * N * H * d, dtype=torch.bfloat16, device="cuda")
    err, raw = cudart.cudaMalloc(in_bytes - 256)  # its own allocation, 256 bytes short
    assert int(err) == 0
    try:
        st = vab.vla_attn_fwd(raw, raw + H * d * 2, raw + 2 * H * d * 2, out, B, N, H, d, 0.125,
                              check=False)
        assert st == vab.ERR_MEMORY
    finally:
        cudart.cudaFree(raw)
    host = torch.empty(B * N * 3 * H * d, dtype=torch.bfloat16)
    hb = host.data_ptr()
    st = vab.vla_attn_fwd(hb, hb + H * d * 2, hb + 2 * H * d * 2, out, B, N, H, d, 0.125,
                          check=False)
    assert st == vab.ERR_MEMORY
    full = torch.empty(B * N * 3 * H * d, dtype=torch.bfloat16, device="cuda")
    fb = full.data_ptr()
    st = vab.vla_attn_fwd(fb, fb + H * d * 2, fb + 2 * H * d * 2, fb, B, N, H, d, 0.125,
                          check=False)
    assert st == vab.ERR_MEMORY  # output overlapping the input
    assert vab.vla_attn_fwd(fb, fb + H * d * 2, fb + 2 * H * d * 2, out, B,
                            vab.vla_attn_max_tokens(d) + 1, H, d, 0.125,
                            check=False) == vab.ERR_UNSUPPORTED
    assert vab.vla_attn_launch_count() >= 0


def test_host_entry_rejects_short_device_buffers_before_copying():
    """vla_attn_fwd_host range-checks qkv_dev and o_dev before it enqueues anything: a
    device input buffer 256 bytes too short for the batch is refused with ERR_MEMORY, no
    kernel is launched and neither the device buffer nor the host output is written."""
    import vit_self_attention_b200 as vab
    from cuda.bindings import runtime as cudart
    B, N, H, d = 2, 50, 12, 64
    in_bytes = B * N * 3 * H * d * 2
    bits = si.packed_qkv(B, N, H, d, seed=777)
    host_in = torch.from_numpy(bits.view(np.int16).copy()).pin_memory()
    host_out = torch.full((B, N, H, d), 0x1234, dtype=torch.int16).pin_memory()
    dev_out = torch.zeros((B, N, H, d), dtype=torch.int16, device="cuda")
    short = in_bytes - 256
    err, raw = cudart.cudaMalloc(short)
    assert int(err) == 0
    try:
        assert int(cudart.cudaMemset(raw, 0x5A, short)[0]) == 0
        torch.cuda.synchronize()
        n0 = vab.vla_attn_launch_count()
        st = vab.vla_attn_fwd_host(host_in, host_out, raw, dev_out, B, N, H, d, 0.125,
                                   check=False)
        torch.cuda.synchronize()
        assert st == vab.ERR_MEMORY
        assert vab.vla_attn_launch_count() == n0
        back = np.empty(short, dtype=np.uint8)
        assert int(cudart.cudaMemcpy(back.ctypes.data, raw, short,
                                     cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost)[0]) == 0
        assert np.all(back == 0x5A), "the short device buffer was written"
        assert bool((host_out == 0x1234).all()), "the host output was written"
        assert bool((dev_out == 0).all())
        # Output overlapping the input is refused too.
        full = torch.empty(in_bytes // 2, dtype=torch.int16, device="cuda")
        st = vab.vla_attn_fwd_host(host_in, host_out, full, full, B, N, H, d, 0.125,
                                   check=False)
        assert st == vab.ERR_MEMORY
    finally:
        cudart.cudaFree(raw)


@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 64), (1, 33, 2, 64), (2, 97, 3, 64), (1, 577, 2, 64),
                                     (1, 50, 2, 72), (2, 113, 3, 72), (10, 700, 16, 64)])
def test_output_stores_stay_inside_the_output(B, N, H, d):
    """The output leaves through TMA stores of 32-row boxes, which overhang the tensor at the
    last rows of every image when N is not a multiple of 32 (or, for whole heads resident
    only without the staging, N=700, through 16-byte row stores): nothing outside
    [B, N, H, d] may be written.  The output is a view into a larger buffer whose guard regions before and
    after it hold a sentinel; they must be unchanged and the output must match the oracle."""
    import vit_self_attention_b200 as vab
    bits = si.packed_qkv(B, N, H, d, seed=4100 + 7 * N + d)
    scale = 1.0 / math.sqrt(d)
    want = oracle.attention_packed_bf16(bits, scale)
    qkv = device_qkv(bits)
    n_o = B * N * H * d
    guard = 8 * 1024  # elements (16 KB) on each side, 16-byte aligned
    sentinel = 0x7FA5
    big = torch.full((guard + n_o + guard,), sentinel, dtype=torch.int16, device="cuda")
    o = big[guard:guard + n_o]
    base = qkv.data_ptr()
    hd = H * d * 2
    vab.vla_attn_fwd(base, base + hd, base + 2 * hd, o.data_ptr(), B, N, H, d, scale)
    torch.cuda.synchronize()
    assert bool((big[:guard] == sentinel).all()), "written before the output"
    assert bool((big[guard + n_o:] == sentinel).all()), "written after the output"
    got = o.view(torch.bfloat16).float().cpu().numpy().astype(np.float64).reshape(B, N, H, d)
    assert_parity(got, want, f"guarded B={B} N={N} H={H} d={d}")
