"""Thread roles and named barriers of the tcgen05 kernels, checked on the CPU.

A named barrier (``bar.sync id, count``) cannot time out: if more or fewer
threads than ``count`` reach it, the block hangs.  These tests read the
kernels' own source, evaluate their compile-time constants and the role
dispatch conditions for every thread of the block, and check that:
  * every thread takes at most one role of the dispatch chain;
  * each ``named_bar_sync(id, count)`` is reached by exactly ``count``
    threads -- those of the role (or prologue) block that contains it;
  * MMA issuers are one thread per dequant group, mapped one to one;
  * the shared-memory table fill covers every entry exactly once.
The conditions are taken from the source text, so a change to the dispatch
is checked as it stands."""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(__file__), "..", "bit_rotated_weight_b200", "csrc")


def _read(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


_CONST = re.compile(r"^\s*constexpr int (\w+) = ([^;]+);", re.M)
_SAFE = re.compile(r"^[\w\s+\-*/()]+$")


def _constants(*sources):
    env = {}
    for src in sources:
        for name, expr in _CONST.findall(src):
            expr = expr.split("//")[0].strip()
            if not _SAFE.match(expr):
                continue
            try:
                env[name] = int(eval(expr.replace("/", "//"), {"__builtins__": {}}, dict(env)))
            except (NameError, SyntaxError):
                pass
    return env


def _to_py(cond):
    cond = cond.replace("&&", " and ").replace("||", " or ")
    assert "!" not in cond.replace("!=", ""), cond
    return cond


def _kernel_lines(src, marker):
    """Lines of the kernel whose definition starts at ``marker`` (up to the
    closing brace at column 0)."""
    lines = src.splitlines()
    start = next(i for i, l in enumerate(lines) if marker in l)
    end = next(i for i in range(start + 1, len(lines)) if lines[i].startswith("}"))
    return lines, start, end


_TOP_IF = re.compile(r"^  if \((.*)\) \{\s*$")
_TOP_ELSE_IF = re.compile(r"^  \} else if \((.*)\) \{\s*$")


def _dispatch(lines, start, end):
    """(head line, [(line, condition)]) of the role chain: the last top-level
    ``if (...) {`` before the first top-level ``} else if``, and its arms."""
    first_else = next(i for i in range(start, end) if _TOP_ELSE_IF.match(lines[i]))
    head = max(i for i in range(start, first_else) if _TOP_IF.match(lines[i]))
    arms = [(head, _TOP_IF.match(lines[head]).group(1))]
    i = head + 1
    while i < end:
        m = _TOP_ELSE_IF.match(lines[i])
        if m:
            arms.append((i, m.group(1)))
        elif lines[i].startswith("  }") and not lines[i].startswith("  } else"):
            return arms, i
        i += 1
    raise AssertionError("role chain not closed")


def _role_of(arms, env, warp, lane, fused):
    for idx, (_, cond) in enumerate(arms):
        if eval(_to_py(cond), {"__builtins__": {}}, dict(env, warp=warp, lane=lane, fused=fused)):
            return idx
    return None


def _block_end(lines, i):
    """End line of the top-level block opened at line i."""
    for j in range(i + 1, len(lines)):
        if lines[j].startswith("  }"):
            return j
    raise AssertionError


_BAR = re.compile(r"named_bar_sync\(([^,()]+),\s*([^()]+)\)")


def _eval_int(expr, env):
    assert _SAFE.match(expr), expr
    return int(eval(expr.replace("/", "//"), {"__builtins__": {}}, dict(env)))


def _check_kernel(src_name, marker, extra_sources=(), fused_values=(False, True)):
    src = _read(src_name)
    env = _constants(*[_read(s) for s in extra_sources], src)
    threads = env["kThreads"]
    assert threads % 32 == 0 and threads <= 1024
    lines, start, end = _kernel_lines(src, marker)
    assert "__launch_bounds__(kThreads" in lines[start]
    arms, chain_end = _dispatch(lines, start, end)
    # other top-level conditional blocks (set-up, prologue)
    blocks = [(i, _TOP_IF.match(lines[i]).group(1), _block_end(lines, i))
              for i in range(start, end) if _TOP_IF.match(lines[i]) and i != arms[0][0]]
    bars = [(i, m.group(1), m.group(2)) for i in range(start, end) for m in _BAR.finditer(lines[i])]
    assert bars, "no named barriers found"
    for fused in fused_values:
        roles = {}
        for tid in range(threads):
            r = _role_of(arms, env, tid // 32, tid % 32, fused)
            roles.setdefault(r, []).append(tid)
        for line, bar_id, bar_cnt in bars:
            cnt = _eval_int(bar_cnt, env)
            assert _eval_int(bar_id, env) != 0, "barrier 0 is __syncthreads"
            # innermost enclosing block: a chain arm or another top-level block
            arm = max((k for k, (l0, _) in enumerate(arms) if l0 < line), default=None)
            in_chain = arm is not None and line < chain_end
            if in_chain:
                n = len(roles.get(arm, []))
            else:
                enclosing = [b for b in blocks if b[0] < line < b[2]]
                assert enclosing, f"{src_name}:{line + 1} named barrier outside any role block"
                l0, cond, _ = max(enclosing)
                n = sum(1 for tid in range(threads)
                        if eval(_to_py(cond), {"__builtins__": {}},
                                dict(env, warp=tid // 32, lane=tid % 32, fused=fused)))
                if n == 0:
                    continue   # the block does not run in this mode
            assert n == cnt, (f"{src_name}:{line + 1}: named_bar_sync({bar_id}, {bar_cnt}) "
                              f"reached by {n} threads (fused={fused})")
    return env, arms, lines


def test_streamk_roles_and_named_barriers():
    env, arms, lines = _check_kernel("tq4_streamk.cu", "__launch_bounds__(kThreads, 1)",
                                     extra_sources=("tq4_internal.h",))
    # role sizes: producer warp, 4 dequant groups of 128 rows, one issuer per
    # group, 128 epilogue threads (one per tensor-memory lane)
    counts = {}
    for tid in range(env["kThreads"]):
        r = _role_of(arms, env, tid // 32, tid % 32, True)
        counts[r] = counts.get(r, 0) + 1
    assert len(arms) == 4
    assert counts[0] == 32
    assert counts[1] == 128 * env["kDequantGroups"]
    assert counts[2] == env["kDequantGroups"]
    assert counts[3] == 128


def test_streamk_issuers_map_one_to_one_onto_groups():
    src = _read("tq4_streamk.cu")
    env = _constants(_read("tq4_internal.h"), src)
    m = re.search(r"int issuer_group\(int warp\) \{ return (.*?); \}", src)
    assert m, "issuer_group not found"
    expr = m.group(1)
    # C conditional -> Python
    c = re.match(r"(.*?) \? (.*?) : (.*)", expr)
    issuers = [w for w in range(env["kThreads"] // 32) if w == 1 or w >= env["kFirstIssuerWarp"]]
    groups = [eval(c.group(2) if eval(c.group(1), {}, dict(env, warp=w)) else c.group(3), {}, dict(env, warp=w))
              for w in issuers]
    assert sorted(groups) == list(range(env["kDequantGroups"]))


def test_streamk_prologue_barrier_and_arrivals():
    src = _read("tq4_streamk.cu")
    env = _constants(_read("tq4_internal.h"), src)
    # the prologue's mbarrier expects one arrival per prologue warp (lane 0)
    assert "mbar_init(&sh.xready, kPrologueThreads / 32);" in src
    assert "if (lane == 0) mbar_arrive(&sh.xready);" in src
    assert env["kPrologueThreads"] % 32 == 0
    warps = [w for w in range(env["kThreads"] // 32)
             if env["kFirstDequantWarp"] <= w < env["kFirstEpilogueWarp"] + 4]
    assert len(warps) * 32 == env["kPrologueThreads"]


def test_streamk_table_fill_covers_each_entry_once():
    src = _read("tq4_streamk.cu")
    env = _constants(_read("tq4_internal.h"), src)
    m = re.search(r"for \(int i = threadIdx\.x - (\d+); warp >= (\d+) && i < ([\w *]+); i \+= kThreads - (\d+)\)", src)
    assert m, "table fill loop not found"
    off, wmin, lim, step_off = int(m.group(1)), int(m.group(2)), eval(m.group(3), {}, env), int(m.group(4))
    seen = {}
    for tid in range(env["kThreads"]):
        if tid // 32 < wmin:
            continue
        i = tid - off
        while i < lim:
            seen[i] = seen.get(i, 0) + 1
            i += env["kThreads"] - step_off
    assert sorted(seen) == list(range(lim)) and set(seen.values()) == {1}
    assert lim * 4 == env["kLutBytes"]


def test_streamk_shared_memory_and_tensor_memory_budgets():
    env = _constants(_read("tq4_internal.h"), _read("tq4_streamk.cu"))
    smem = env["kStages"] * (env["kCodesBytes"] + env["kXBytes"]) + env["kLutBytes"]
    assert smem + 1024 <= 227 * 1024
    # cluster split-K: the owner CTA's reduction buffer (codes of the stages
    # fused mode never loads) holds s partials of 32 token rows x ceil(128/s)
    # weight rows, for every split s in [2, 8]
    assert env["kRedOff"] == env["kFusedMaxIters"] * env["kCodesBytes"]
    room = env["kStages"] * env["kCodesBytes"] - env["kRedOff"]
    for s in range(2, 9):
        assert s * env["kSegRows"] * (-(-128 // s)) * 4 <= room
    assert env["kTmemCols"] <= 512


def test_gemm_roles_and_named_barriers():
    env, arms, _ = _check_kernel("tq4_gemm.cu", "__launch_bounds__(kThreads, 1)", fused_values=(False,))
    counts = {}
    for tid in range(env["kThreads"]):
        r = _role_of(arms, env, tid // 32, tid % 32, False)
        counts[r] = counts.get(r, 0) + 1
    assert counts[len(arms) - 1] == 128   # epilogue: one thread per tensor-memory lane


def test_streamk_resident_stage_release_has_no_second_waiter():
    # With the resident x' a codes stage is released by the dequant warps as
    # soon as they read it (4 arrivals), so it may be refilled before the
    # group's issuer gets to that iteration: the issuer must not wait on the
    # stage's `full` barrier then (its parity wait could be two phases
    # behind).  The refill waits for the dequant warps, not the MMAs.
    src = _read("tq4_streamk.cu")
    assert "mbar_init(&sh.done[i - kStages], a.x_resident ? 4 : 1)" in src
    assert "if (!resident && !mbar_wait(&sh.full[s], (li / kStages) & 1, abortp)) {" in src
    assert "if (!resident) mma_commit(&sh.done[s]);" in src


def test_streamk_overflowing_levels_fall_back_to_the_exact_path():
    # a half-block scale above ~93.6 overflows the fp16 levels: the epilogue
    # detects the non-finite sums (one NaN test over v * 0) and recomputes the
    # row's portion with fp32 levels, reading x' from memory or, in fused
    # mode, from the B tiles; no kernel raises the scale-range status any more
    src = _read("tq4_streamk.cu")
    assert "z = __fmaf_rn(v[j], 0.0f, z);" in src and "const bool bad = z != z;" in src
    assert "exact_row_portion(a.codes + wrow * (a.k / 2), a.scales + wrow * (a.k / 16), kc0, kc1," in src
    assert "a.xr ? a.xr + static_cast<int64_t>(sg.row0) * a.k : nullptr" in src
    for name in ("tq4_streamk.cu", "tq4_decode.cu", "tq4_kernels.cu", "tq4_gemm.cu", "tq4_api.cu", "tq4_static.cu"):
        assert "raise_status(TQ_DEV_SCALE_RANGE)" not in _read(name), name
    api = _read("tq4_api.cu") + _read("tq4_static.cu")
    assert api.count("a.codes = w->codes;") == 2 and "a.xr = fused ? nullptr : xr;" in api
    assert "a.codes = up->codes;" in api and "b.codes = down->codes;" in api
    assert "a.xr = xr;" in api and "b.xr = hr;" in api


def test_quantize_fast_path_matches_the_checked_forms():
    # the bucket search and the quotient sequence are the forms that
    # test_abi_host.py (exhaustively on the threshold buckets) and the GPU
    # probe of the division checked: the table as built there, the search
    # only on symmetric thresholds with one per bucket and on finite half
    # blocks; other half blocks keep the division and the full search
    src = _read("tq4_kernels.cu")
    for s in ("constexpr int kQBucket0 = 122 << 4;",
              "constexpr int kQBuckets = 130;",
              "const float lo = i == 0 ? 0.0f : __uint_as_float(static_cast<uint32_t>(kQBucket0 + i - 1) << 19);",
              "const float hi = i == kQBuckets - 1 ? INFINITY : __uint_as_float(static_cast<uint32_t>(kQBucket0 + i) << 19);",
              "th.bucket[i] = make_uint2(inside, below);",
              "fast = fast && bucket_of(cb.thresholds[8 + j]) != bucket_of(cb.thresholds[9 + j]);",
              "int q = static_cast<int>(ab >> 19) - (kQBucket0 - 1);",
              "q = q < 0 ? 0 : (q > kQBuckets - 1 ? kQBuckets - 1 : q);",
              "const uint32_t c = e.y + ((ab + (pos ? 0u : 1u) > e.x) ? 1u : 0u);",
              "code = pos ? 8u + c : 7u - c;",
              "if (fin && d != 0.0f) {",
              "const float y = __frcp_rn(d);",
              "const float u = __fmaf_rn(__fmaf_rn(-q, d, a[16 * h + i]), y, q);",
              "const float u = __fdiv_rn(a[16 * h + i], d);",
              "if (!finite) raise_status(TQ_DEV_NONFINITE);",
              "__syncwarp();   // every lane is done with the tile (the check above reads it)"):
        assert s in src, s


def test_streamk_exact_path_reads_x_where_the_fused_prologue_wrote_it():
    # In fused mode x' lives only in the CTA's B tiles.  The prologue writes
    # unit u = (iteration li, slice sl, token j) as four 16-byte chunks q at
    # btile(li) + (sl >> 1) * kXHalfBytes + 128 j + ((q ^ cx) << 4), with
    # cx = 4 (sl & 1) ^ (j & 7), element t of chunk q at byte 2 t.  The exact
    # fallback of the epilogue reads column kk of local iteration li at the
    # address below.  Both as written in the source, and the same byte for
    # every (li, sl, j, q, t).
    src = _read("tq4_streamk.cu")
    assert "cx = ((sl & 1) * 4) ^ (j & 7);   // chunk q sits at chunk q ^ cx" in src
    assert "return btile_of(li) + (sl >> 1) * kXHalfBytes + j * 128;" in src
    assert "*reinterpret_cast<uint4*>(rowp + ((q ^ cx) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);" in src
    assert ": *reinterpret_cast<const uint16_t*>(xs + li * kXBytes + (e >> 6) * kXHalfBytes + jj * 128 +" in src
    assert "((((e64 >> 3) ^ (jj & 7))) << 4) + (e64 & 7) * 2);" in src
    assert "const int li = li0 + (kk >> 7) - (kc0 >> 7), e = kk & 127, e64 = e & 63;" in src
    env = _constants(_read("tq4_internal.h"), src)
    half, full = env["kXHalfBytes"], env["kXBytes"]
    for li in range(env["kFusedMaxIters"]):
        for sl in range(4):
            for j in range(env["kSegRows"]):
                cx = ((sl & 1) * 4) ^ (j & 7)
                for q in range(4):
                    for t in range(8):
                        written = li * full + (sl >> 1) * half + j * 128 + ((q ^ cx) << 4) + 2 * t
                        e = 32 * sl + 8 * q + t
                        e64 = e & 63
                        read = li * full + (e >> 6) * half + j * 128 + (((e64 >> 3) ^ (j & 7)) << 4) + (e64 & 7) * 2
                        assert written == read, (li, sl, j, q, t)
