"""Host-only checks of libq4dec: it loads, exports every symbol the header
declares, validates arguments before touching CUDA, and plans launches."""
import ctypes
import os
import re

import pytest

from bit_weight_streaming_dequant_b200 import q4dec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q4dec.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(q[48][a-z0-9_]*)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    L = q4dec.lib()
    declared = _declared_functions()
    assert set(declared) == set(q4dec.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def test_version_and_status_strings():
    L = q4dec.lib()
    assert L.q4d_version() == 20000
    for code in range(8):
        assert L.q4d_status_string(code) != b"unknown status"
    assert L.q4d_status_string(99) == b"unknown status"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("M,N,K,code", [
    (0, 16, 256, 2), (6, 16, 256, 2), (1, 16, 100, 2), (1, 16, 0, 2),
    (1, 0, 256, 1), (1, -3, 256, 1), (1, 16, -256, 1),
])
def test_gemv_rejects_bad_shapes_without_cuda(M, N, K, code):
    L = q4dec.lib()
    assert L.q4_gemv_ex(FAKE, FAKE, FAKE, M, N, K, None, None, 0) == code
    assert L.q4_gemv(FAKE, FAKE, FAKE, M, N, K) == code


def test_gemv_ex2_rejects_unknown_flags_and_bad_shapes_without_cuda():
    L = q4dec.lib()
    for flags in (4, 0x80000000, 5, 7):
        assert L.q4_gemv_ex2(FAKE, FAKE, FAKE, 1, 16, 256, None, None, 0, flags) == 1
        assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE, 1, 16, 256, None, None, 0, flags) == 1
    bf16 = q4dec.GEMV_OUT_BF16
    for flags in (0, q4dec.GEMV_WEIGHT_PREFETCH, bf16, bf16 | q4dec.GEMV_WEIGHT_PREFETCH):
        assert L.q4_gemv_ex2(FAKE, FAKE, FAKE, 6, 16, 256, None, None, 0, flags) == 2
        assert L.q4_gemv_ex2(FAKE + 8, FAKE, FAKE, 1, 16, 256, None, None, 0, flags) == 3
        assert L.q4_gemv_ex2(None, FAKE, FAKE, 1, 16, 256, None, None, 0, flags) == 1
        # y: 4-byte alignment for fp32 outputs, 2-byte for bf16
        assert L.q4_gemv_ex2(FAKE, FAKE, FAKE + 1, 1, 16, 256, None, None, 0, flags) == 3
        assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE + 1, 1, 16, 256, None, None, 0, flags) == 3
    for flags in (0, q4dec.GEMV_WEIGHT_PREFETCH):
        assert L.q4_gemv_ex2(FAKE, FAKE, FAKE + 2, 1, 16, 256, None, None, 0, flags) == 3


def test_gemv_rejects_null_and_misaligned_pointers():
    L = q4dec.lib()
    assert L.q4_gemv_ex(None, FAKE, FAKE, 1, 16, 256, None, None, 0) == 1
    assert L.q4_gemv_ex(FAKE, None, FAKE, 1, 16, 256, None, None, 0) == 1
    assert L.q4_gemv_ex(FAKE, FAKE, None, 1, 16, 256, None, None, 0) == 1
    assert L.q4_gemv_ex(FAKE + 8, FAKE, FAKE, 1, 16, 256, None, None, 0) == 3
    assert L.q4_gemv_ex(FAKE, FAKE + 2, FAKE, 1, 16, 256, None, None, 0) == 3
    assert L.q4_gemv_ex(FAKE, FAKE, FAKE + 2, 1, 16, 256, None, None, 0) == 3
    assert L.q4_gemv_ex(FAKE, FAKE, FAKE, 1, 16, 256, None, FAKE + 4, 64) == 3


@pytest.mark.parametrize("ctx,nq,nkv,hd,M,stride,scale,code", [
    (100, 24, 4, 128, 1, 100, 1.0, 2),    # head_dim != 256
    (100, 24, 5, 256, 1, 100, 1.0, 2),    # n_q % n_kv
    (4, 24, 4, 256, 5, 4, 1.0, 2),        # ctx_len < M
    (100, 24, 4, 256, 6, 100, 1.0, 2),    # M > 5
    (100, 24, 4, 256, 0, 100, 1.0, 2),    # M < 1
    (100, 24, 4, 256, 1, 99, 1.0, 2),     # stride < ctx_len
    (0, 24, 4, 256, 1, 0, 1.0, 1),        # empty context
    (100, 0, 4, 256, 1, 100, 1.0, 1),
    (100, 24, 0, 256, 1, 100, 1.0, 1),
    (100, 24, 4, 256, 1, 100, float("nan"), 1),
    (100, 24, 4, 256, 1, 100, float("inf"), 1),
])
def test_attn_rejects_bad_arguments_without_cuda(ctx, nq, nkv, hd, M, stride, scale, code):
    L = q4dec.lib()
    for fn in (L.q4kv_attn_decode_ex, L.q8kv_attn_decode_ex):
        assert fn(FAKE, FAKE, FAKE, FAKE, ctx, nq, nkv, hd, M, stride,
                  ctypes.c_float(scale), None, None, 0) == code


def test_attn_rejects_null_and_misaligned():
    L = q4dec.lib()
    args = (4096, 24, 4, 256, 1, 4096, ctypes.c_float(1.0), None, None, 0)
    for fn in (L.q4kv_attn_decode_ex, L.q8kv_attn_decode_ex):
        assert fn(None, FAKE, FAKE, FAKE, *args) == 1
        assert fn(FAKE, FAKE, FAKE, None, *args) == 1
        assert fn(FAKE + 8, FAKE, FAKE, FAKE, *args) == 3
        assert fn(FAKE, FAKE + 4, FAKE, FAKE, *args) == 3
        assert fn(FAKE, FAKE, FAKE + 12, FAKE, *args) == 3
        assert fn(FAKE, FAKE, FAKE, FAKE + 1, *args) == 3


def test_q8_plan_and_workspace_queries():
    L = q4dec.lib()
    a = q4dec.AttnPlan()
    assert L.q8kv_plan_attn(4096, 24, 4, 256, 1, 0, ctypes.byref(a)) == 1
    assert L.q8kv_plan_attn(4096, 24, 4, 64, 1, 148, ctypes.byref(a)) == 2
    assert L.q8kv_plan_attn(4096, 24, 4, 256, 1, 148, None) == 1
    assert L.q8kv_attn_workspace_bytes(4096, 24, 4, 64, 1) == 0       # invalid shape
    # one row per CTA still takes the tensor-memory kernel (448 threads)
    assert L.q8kv_plan_attn(4096, 4, 4, 256, 1, 148, ctypes.byref(a)) == 0
    assert a.threads == 448 and a.tile_tokens == 128


def test_plan_rejects_bad_inputs():
    L = q4dec.lib()
    p = q4dec.GemvPlan()
    assert ctypes.sizeof(p) == 8 * 4 + 2 * 8
    assert L.q4d_plan_gemv(1, 16, 256, 0, ctypes.byref(p)) == 1
    assert L.q4d_plan_gemv(1, 16, 256, 148, None) == 1
    assert L.q4d_plan_gemv(7, 16, 256, 148, ctypes.byref(p)) == 2
    a = q4dec.AttnPlan()
    assert L.q4d_plan_attn(4096, 24, 4, 256, 1, 0, ctypes.byref(a)) == 1
    assert L.q4d_plan_attn(4096, 24, 4, 64, 1, 148, ctypes.byref(a)) == 2


def test_workspace_queries_without_device_use_the_fallback_plan():
    L = q4dec.lib()
    # invalid shapes report 0
    assert L.q4d_gemv_workspace_bytes(0, 16, 256) == 0
    assert L.q4d_attn_workspace_bytes(4096, 24, 5, 256, 1) == 0
    # row blocks shared between CTAs need partial-sum space; one CTA does not;
    # the long context needs merge space
    p = q4dec.plan_gemv(1, 17408, 5120, 148)
    assert L.q4d_gemv_workspace_bytes(1, 17408, 5120) == p.workspace_bytes > 0
    assert L.q4d_gemv_workspace_bytes(1, 1, 256) == 0
    assert L.q4d_attn_workspace_bytes(262144, 24, 4, 256, 5) > 0


def _batch_jobs(n, **kw):
    jobs = (q4dec.GemvJob * n)()
    for i in range(n):
        jobs[i] = q4dec.GemvJob(FAKE, FAKE, FAKE, kw.get("N", 256), kw.get("K", 512),
                                kw.get("flags", 0), kw.get("wait_for", -1 if i == 0 else i - 1))
    return jobs


def test_gemv_batch_prepare_validates_without_cuda():
    L = q4dec.lib()
    n = 3
    nbytes = L.q4d_gemv_batch_desc_bytes(n)
    assert nbytes > 0 and L.q4d_gemv_batch_desc_bytes(0) == 0
    buf = ctypes.create_string_buffer(nbytes)
    ws = ctypes.c_size_t(0)
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n, N=17408, K=5120), n, 1, 148, buf, nbytes,
                                    ctypes.byref(ws)) == 0
    assert ws.value == 3 * q4dec.plan_gemv(1, 17408, 5120, 148).workspace_bytes
    # two row blocks, one CTA each: nothing to share, no workspace
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n), n, 1, 148, buf, nbytes, ctypes.byref(ws)) == 0
    assert ws.value == 0
    # the completion counters at the descriptor's end are handed over zeroed
    assert set(buf.raw[nbytes - 16:]) == {0}
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n), n, 6, 148, buf, nbytes, None) == 2
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n), n, 1, 0, buf, nbytes, None) == 1
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n), n, 1, 148, buf, nbytes - 1, None) == 1
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n, K=100), n, 1, 148, buf, nbytes, None) == 2
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n, flags=1), n, 1, 148, buf, nbytes, None) == 1
    bad = _batch_jobs(n)
    bad[2].wait_for = 2                       # a job cannot wait for itself
    assert L.q4d_gemv_batch_prepare(bad, n, 1, 148, buf, nbytes, None) == 1
    bad = _batch_jobs(n)
    bad[1].x = FAKE + 8                       # activations 16-byte aligned
    assert L.q4d_gemv_batch_prepare(bad, n, 1, 148, buf, nbytes, None) == 3
    bad = _batch_jobs(n)
    bad[0].y = None
    assert L.q4d_gemv_batch_prepare(bad, n, 1, 148, buf, nbytes, None) == 1
    # a launch refuses a foreign or bad descriptor before touching CUDA
    assert L.q4d_gemv_batch_prepare(_batch_jobs(n, N=17408, K=5120), n, 1, 148, buf, nbytes,
                                    ctypes.byref(ws)) == 0
    assert L.q4_gemv_batch_ex(None, FAKE, None, FAKE, 1 << 20, 0) == 1
    assert L.q4_gemv_batch_ex(buf, FAKE, None, FAKE, 1 << 20, 2) == 1
    junk = ctypes.create_string_buffer(nbytes)
    assert L.q4_gemv_batch_ex(junk, FAKE, None, FAKE, 1 << 20, 0) == 1
    assert L.q4_gemv_batch_ex(buf, FAKE + 8, None, FAKE, 1 << 20, 0) == 3
    assert L.q4_gemv_batch_ex(buf, FAKE, None, None, 0, 0) == 4


def test_append_rejects_bad_arguments_without_cuda():
    L = q4dec.lib()
    assert L.q4kv_append(None, FAKE, FAKE, FAKE, 4, 64, 0, 1, None) == 1
    assert L.q4kv_append(FAKE, FAKE, FAKE, FAKE, 0, 64, 0, 1, None) == 1
    assert L.q4kv_append(FAKE, FAKE, FAKE, FAKE, 4, 64, -1, 1, None) == 1
    assert L.q4kv_append(FAKE, FAKE, FAKE, FAKE, 4, 64, 0, 0, None) == 1
    assert L.q4kv_append(FAKE, FAKE, FAKE, FAKE, 4, 64, 60, 5, None) == 2
    assert L.q4kv_append(FAKE + 8, FAKE, FAKE, FAKE, 4, 64, 0, 1, None) == 3
    assert L.q4kv_append(FAKE, FAKE, FAKE + 2, FAKE, 4, 64, 0, 1, None) == 3


def test_swiglu_rejects_bad_arguments_without_cuda():
    L = q4dec.lib()
    assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE, 1, 16, 256, None, None, 0, 4) == 1
    assert L.q4_gemv_swiglu_ex(None, FAKE, FAKE, 1, 16, 256, None, None, 0, 0) == 1
    assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE, 6, 16, 256, None, None, 0, 0) == 2
    assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE, 1, 16, 100, None, None, 0, 0) == 2
    assert L.q4_gemv_swiglu_ex(FAKE, FAKE, FAKE, 1, 0, 256, None, None, 0, 0) == 1
    assert L.q4_gemv_swiglu_ex(FAKE + 8, FAKE, FAKE, 1, 16, 256, None, None, 0, 0) == 3
    # workspace: a plan over 2N rows in pairs
    assert L.q4d_gemv_swiglu_workspace_bytes(1, 8, 65536) > 0
    assert L.q4d_gemv_swiglu_workspace_bytes(1, 0, 256) == 0


def test_wait_selftest_rejects_bad_arguments_without_cuda():
    L = q4dec.lib()
    assert L.q4d_wait_selftest(None, 1000, 0, None) == 1
    assert L.q4d_wait_selftest(FAKE, 0, 0, None) == 1
    assert L.q4d_wait_selftest(FAKE, 10_000_001, 0, None) == 1
    assert L.q4d_wait_selftest(FAKE + 2, 1000, 0, None) == 3


def _contributors(rbs, upr, U, G):
    slots = 0
    for rb in range(rbs):
        first = ((rb * upr + 1) * G - 1) // U
        last = ((rb * upr + upr) * G - 1) // U
        if last > first:
            slots = max(slots, last - first + 1)
    return slots


@pytest.mark.parametrize("M,sms", [(1, 148), (5, 148), (3, 132)])
def test_gemv_batch_descriptor_matches_the_planning_model(M, sms):
    # a decode-like batch (two layers of gate, up, down, in, out; a fused gate /
    # up job; a tiny job) prepared on the host and read back field by field:
    # header, then one job descriptor per job (pointers, rows, K / 256, flags,
    # wait_for, row blocks, units per row block, units, CTAs, partial slots,
    # rotation, partial-slot offset), against a plain model of the partition
    import struct
    shapes = [(17408, 5120, 0), (17408, 5120, 0), (5120, 17408, 0), (6144, 5120, 0),
              (5120, 6144, 0)] * 2 + [(1024, 5120, q4dec.GEMV_SWIGLU), (37, 256, 2)]
    n = len(shapes)
    jobs = (q4dec.GemvJob * n)()
    for i, (N, K, fl) in enumerate(shapes):
        jobs[i] = q4dec.GemvJob(FAKE + 16 * i, FAKE + 32 * i, FAKE + 64 * i, N, K, fl, i - 1)
    L = q4dec.lib()
    nbytes = L.q4d_gemv_batch_desc_bytes(n)
    buf = ctypes.create_string_buffer(nbytes)
    ws = ctypes.c_size_t(0)
    assert L.q4d_gemv_batch_prepare(jobs, n, M, sms, buf, nbytes, ctypes.byref(ws)) == 0
    raw = buf.raw
    magic, n_jobs, M_h, sms_h, grid = struct.unpack_from("<Iiiii", raw, 0)
    assert (n_jobs, M_h, sms_h) == (n, M, sms) and magic != 0
    (ws_bytes,) = struct.unpack_from("<Q", raw, 24)
    assert ws_bytes == ws.value
    model, units_before, entries, launch_grid = [], 0, 0, 1
    for N, K, fl in shapes:
        rows = 2 * N if fl & q4dec.GEMV_SWIGLU else N
        rbs, upr = -(-rows // 128), -(-(K // 256) // 2)
        launch_grid = max(launch_grid, min(sms, rbs * upr))
    assert grid == launch_grid
    for i, (N, K, fl) in enumerate(shapes):
        rows = 2 * N if fl & q4dec.GEMV_SWIGLU else N
        rbs, upr = -(-rows // 128), -(-(K // 256) // 2)
        U = rbs * upr
        G = min(launch_grid, U)
        slots = _contributors(rbs, upr, U, G)
        off = 64 + i * 80
        W, x, y, part_off = struct.unpack_from("<QQQq", raw, off)
        (Nd, nsb, flags, wait_for, rbs_d, upr_d, units, G_d, slots_d, rot) = \
            struct.unpack_from("<10i", raw, off + 32)
        (w_bytes,) = struct.unpack_from("<q", raw, off + 72)
        assert w_bytes == rows * (K // 256) * 144  # the index checks' weight extent
        assert (W, x, y) == (FAKE + 16 * i, FAKE + 32 * i, FAKE + 64 * i)
        assert (Nd, nsb, wait_for) == (rows, K // 256, i - 1)
        assert bool(flags & 2) == bool(fl & q4dec.GEMV_SWIGLU) and bool(flags & 1) == bool(fl & 2)
        assert (rbs_d, upr_d, units, G_d, slots_d) == (rbs, upr, U, G, slots)
        assert rot == units_before % launch_grid
        assert part_off == entries
        units_before += U
        entries += rbs * slots * M * 128 if slots else 0
    assert ws.value == entries * 8
    # the completion counters after the jobs are zero as prepared
    assert set(raw[64 + n * 80:nbytes]) == {0}


# ---- the debug build (libq4dec_debug.so: the same sources with Q4D_DEBUG)

def _debug_lib():
    assert os.path.exists(q4dec.DEBUG_LIB_PATH), "libq4dec_debug.so is built beside libq4dec.so"
    D = ctypes.CDLL(q4dec.DEBUG_LIB_PATH)
    D.q4d_debug_build.restype = ctypes.c_int
    D.q4d_debug_limit_weights.argtypes = [ctypes.c_ulonglong]
    D.q4d_debug_limit_weights.restype = ctypes.c_int
    D.q4d_gemv_batch_desc_bytes.argtypes = [ctypes.c_int]
    D.q4d_gemv_batch_desc_bytes.restype = ctypes.c_size_t
    D.q4d_gemv_batch_prepare.argtypes = [ctypes.POINTER(q4dec.GemvJob), ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]
    D.q4d_gemv_batch_prepare.restype = ctypes.c_int
    D.q4d_index_check_selftest.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                                           ctypes.c_void_p]
    D.q4d_index_check_selftest.restype = ctypes.c_int
    return D


def test_debug_library_exports_every_declared_function_and_says_it_is_the_debug_build():
    D = _debug_lib()
    for name in _declared_functions():
        assert hasattr(D, name), name
    assert D.q4d_debug_build() == 1
    assert q4dec.lib().q4d_debug_build() == 0


def test_index_check_selftest_validates_before_launching():
    for L in (q4dec.lib(), _debug_lib()):
        assert L.q4d_index_check_selftest(None, 0, 1, None) == 1
        assert L.q4d_index_check_selftest(FAKE, 0, -1, None) == 1
        assert L.q4d_index_check_selftest(FAKE, 0, 65, None) == 1
        assert L.q4d_index_check_selftest(FAKE + 2, 0, 1, None) == 3


def test_weight_limit_is_a_debug_build_hook_and_caps_the_declared_extent():
    import struct
    assert q4dec.lib().q4d_debug_limit_weights(4096) == 1  # release: refused, nothing set
    D = _debug_lib()
    shapes = [(512, 1024), (16, 256)]                       # 294912 and 2304 bytes of weights
    jobs = (q4dec.GemvJob * 2)()
    for i, (N, K) in enumerate(shapes):
        jobs[i] = q4dec.GemvJob(FAKE, FAKE, FAKE, N, K, 0, -1)
    nbytes = D.q4d_gemv_batch_desc_bytes(2)
    for limit, expect in ((4096, [4096, 2304]), (0, [294912, 2304])):
        assert D.q4d_debug_limit_weights(limit) == 0
        buf = ctypes.create_string_buffer(nbytes)
        ws = ctypes.c_size_t(0)
        assert D.q4d_gemv_batch_prepare(jobs, 2, 1, 148, buf, nbytes, ctypes.byref(ws)) == 0
        got = [struct.unpack_from("<q", buf.raw, 64 + i * 80 + 72)[0] for i in range(2)]
        assert got == expect
    assert D.q4d_debug_limit_weights(0) == 0


def _kernel_sources():
    csrc = os.path.join(ROOT, "bit_weight_streaming_dequant_b200", "csrc")
    return {n: open(os.path.join(csrc, n)).read() for n in sorted(os.listdir(csrc))
            if n.endswith(".cuh") and n != "q4dec_device.cuh"}


def test_every_bulk_copy_and_global_store_of_the_kernels_is_index_checked():
    """Each bulk copy's source and each plain global store of the kernels is
    guarded by an index check within the few lines before it (a lint: the
    debug-build parity runs show that no check fails on valid inputs)."""
    guards = ("Q4D_CHECK", "_in_range", "x_offset_m<")
    stores = re.compile(r"\b(a\.out|a\.ws_o|a\.ws_ml|sb)\[[^\]]*\]\s*=[^=]|store_out\(J->y|"
                        r"st_relaxed_gpu_u64\(s_e|s_e\[seg_index\([^)]*\)\]\s*=|"
                        r"reinterpret_cast<__half\*>\(sb")
    for name, text in _kernel_sources().items():
        lines = text.splitlines()
        for i, line in enumerate(lines):
            code = line.split("//")[0]
            if re.search(r"\bbulk_g2s(_nohint)?\(", code) and "__device__" not in code:
                window = "\n".join(lines[max(0, i - 12):i + 2])
                assert any(g in window for g in guards), f"{name}:{i + 1}: {line.strip()}"
            if stores.search(code):
                window = "\n".join(lines[max(0, i - 6):i + 1])
                assert any(g in window for g in guards), f"{name}:{i + 1}: {line.strip()}"


def test_check_sites_of_the_binding_match_the_device_enum():
    # the site numbers the binding names are the kernels' IndexCheckSite values
    text = open(os.path.join(ROOT, "bit_weight_streaming_dequant_b200", "csrc",
                             "q4dec_device.cuh")).read()
    body = text[text.index("enum IndexCheckSite"):]
    body = body[:body.index("};")]
    sites = {int(v) for v in re.findall(r"kSite\w+\s*=\s*(\d+)", body)}
    assert sites == set(q4dec.CHECK_SITES)
    assert q4dec.STATUS[7] == "Q4D_ERR_DEVICE_INDEX"
    header = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    assert re.search(r"Q4D_ERR_DEVICE_INDEX\s*=\s*7", header)


def test_use_debug_library_switches_the_loaded_library_and_back():
    try:
        assert q4dec.use_debug_library(True) == q4dec.DEBUG_LIB_PATH
        assert q4dec.debug_build()
        assert q4dec.use_debug_library(False) == q4dec.RELEASE_LIB_PATH
        assert not q4dec.debug_build()
    finally:
        q4dec.use_debug_library(False)
