"""Mutation check of the oracle's pins and of the benchmark's host
arithmetic (not collected by pytest; run by hand).

    python tests/mutation_check.py [mutation name ...]

Each entry below plants one plausible mistake: in the oracle (M: a dropped
term, a wrong sign, index or axis, an off-by-one, a wrong tie-break or
reading), in bench.py's host logic (BENCH: the pair count, the roofline
arithmetic, the sample extrapolation, the traffic digest, clock parsing,
rank reductions), in the binding's checks (BINDING) or in the C ABI's
argument validation (CABI; the copy's library is rebuilt for each).  For each entry the script copies the repository into a
temporary directory, applies the mutation to the copy and runs the CPU
suite (-m "not gpu", stopping at the first failure) on the copy.  A mutation
that no test catches marks a missing test.  The repository itself is never
modified.  A full run takes about 30 minutes on 8 cores; it exits 1 if any
mutation survives.
"""
import os
import shutil
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

M = [
 ("r_v sample variance", "sig2[:, d] = ((prof - mu) ** 2).mean(axis=1).mean(axis=1)", "sig2[:, d] = ((prof - mu) ** 2).sum(axis=1).mean(axis=1) / (ZONE - 1)"),
 ("H profile pools the wrong axes", "prof_H = v.mean(axis=(1, 3))", "prof_H = v.mean(axis=(1, 2))"),
 ("spatial term around the zone mean", "spatial = ((v - prof_T[:, :, None, None, :]) ** 2)", "spatial = ((v - v.mean(axis=(1, 2, 3), keepdims=True)) ** 2)"),
 ("temporal term over 8 not 7", "temporal = (diff ** 2).sum(axis=1).mean(axis=1) / (ZONE - 1)", "temporal = (diff ** 2).sum(axis=1).mean(axis=1) / ZONE"),
 ("temporal term abs not square", "temporal = (diff ** 2).sum(axis=1)", "temporal = np.abs(diff).sum(axis=1)"),
 ("a2v norm L1", "return np.sqrt((h * h).sum(axis=1))", "return np.abs(h).sum(axis=1)"),
 ("a2v norm without sqrt", "return np.sqrt((h * h).sum(axis=1))", "return (h * h).sum(axis=1)"),
 ("a2v profiles swapped", "for d, ax in enumerate(((2, 3), (1, 3), (1, 2))):", "for d, ax in enumerate(((1, 3), (2, 3), (1, 2))):"),
 ("abar from zone max", "abar_raw = z.mean(axis=(1, 2, 3))", "abar_raw = z.max(axis=(1, 2, 3))"),
 ("zero-variance shares 0", "out = np.full_like(sig2, 1.0 / 3.0)", "out = np.zeros_like(sig2)"),
 ("eps dropped", "    return g + eps", "    return g"),
 ("abar not applied", "g = g + abar[:, None] * vhat", "g = g + vhat"),
 ("normalise by sum", "    return x / m\n", "    return x / x.sum()\n"),
 ("threshold strict", "B = np.where(rho >= tau128, 64, np.where(rho >= tau256, 128, 256))", "B = np.where(rho > tau128, 64, np.where(rho > tau256, 128, 256))"),
 ("volumes reversed", "B = np.where(rho >= tau128, 64, np.where(rho >= tau256, 128, 256))", "B = np.where(rho >= tau128, 256, np.where(rho >= tau256, 128, 64))"),
 ("lstar sign", "return -alpha * lg + (S[..., None]", "return alpha * lg + (S[..., None]"),
 ("lstar over 2", "alpha * lg.sum(axis=-1, keepdims=True)) / 3.0", "alpha * lg.sum(axis=-1, keepdims=True)) / 2.0"),
 ("lstar natural log of B", "S = np.log2(B.astype(np.float64))", "S = np.log(B.astype(np.float64))"),
 ("lstar shift ignores alpha", "(S[..., None] + alpha * lg.sum(", "(S[..., None] + 0.5 * lg.sum("),
 ("shape tie to highest id", "            if dist < best:\n                second, best, best_id", "            if dist <= best:\n                second, best, best_id"),
 ("shape distance L1", "dist = sum((l[d] - ls[idx][d]) ** 2 for d in range(3))", "dist = sum(abs(l[d] - ls[idx][d]) for d in range(3))"),
 ("block tokens y fastest", "return ((t * H + y) * W + x).reshape(-1)", "return ((t * H + y) * W + x).transpose(0, 2, 1).reshape(-1)"),
 ("zones zT fastest", "perm = (0, 2, 4, 1, 3, 5)", "perm = (4, 2, 0, 1, 3, 5)"),
 ("candidate order reversed", "        for bT in (2, 4, 8):", "        for bT in (8, 4, 2):"),
 ("block mean over B-1", "out[bl] = acc * np.float32(1.0 / B)", "out[bl] = acc * np.float32(1.0 / (B - 1))"),
 ("score scale dropped", "    return acc * np.float32(scale)", "    return acc"),
 ("top-k floor", "int(math.ceil(float(np.float32(topk_frac)) * nb))", "int(math.floor(float(np.float32(topk_frac)) * nb))"),
 ("top-p strict", "hit = np.nonzero(csum >= target)[0]", "hit = np.nonzero(csum > target)[0]"),
 ("top-p crossing dropped", "n_p = int(hit[0]) + 1 if hit.size else nb", "n_p = int(hit[0]) if hit.size else nb"),
 ("ties by index descending", "order = np.lexsort((j, -s))", "order = np.lexsort((-j, -s))"),
 ("intersection not union", "    n = max(k, n_p)", "    n = min(k, n_p)"),
 ("p >= 1 rule dropped", "    elif p >= 1:\n        n_p = nb", "    elif p > 1:\n        n_p = nb"),
 ("fwd scale dropped", "    s = (q @ k.T) * scale\n    m = s.max", "    s = (q @ k.T)\n    m = s.max"),
 ("lse without the max", "lse = (m + np.log(l))[:, 0]", "lse = np.log(l)[:, 0]"),
 ("bwd dS sign", "dS = P * (dP - Dq)", "dS = P * (Dq - dP)"),
 ("bwd dK scale dropped", "np.add.at(dK[:, h], keys, scale * (dS.T @ q))", "np.add.at(dK[:, h], keys, dS.T @ q)"),
 ("bwd Delta from dO.dO", "Dq = (P * dP).sum(axis=1, keepdims=True)", "Dq = (do * do).sum(axis=1, keepdims=True)"),
 ("bwd dQ scale dropped", "dQ[qi, h] += scale * (dS @ k)", "dQ[qi, h] += dS @ k"),
 ("guidance bits swapped", "video=not (guidance & 1), audio=not (guidance & 2)", "video=not (guidance & 2), audio=not (guidance & 1)"),
 ("density modes swapped", "    if mode == 1:\n        return spatial", "    if mode == 1:\n        return temporal"),
 ("vhat not normalised", "        vhat = shares(sig2a)", "        vhat = sig2a"),
 ("rho per all heads", "        rho = normalise_by_max(density_raw(spatial, temporal, abar_raw, density))", "        rho = density_raw(spatial, temporal, abar_raw, density) / 1.0"),
 ("abar not normalised in the plan", "        abar = normalise_by_max(abar_raw)", "        abar = abar_raw"),
 ("selection in score order", "    return np.sort(order[:n]), dict(", "    return order[:n], dict("),
 ("temporal term over row means", "diff = prof_T[:, 1:, :] - prof_T[:, :-1, :]", "diff = prof_H[:, 1:, :] - prof_H[:, :-1, :]"),
 ("permutation inverted", "        perm[p0:p0 + B] = block_tokens(T, H, W, t0, y0, x0, sid)", "        perm[block_tokens(T, H, W, t0, y0, x0, sid)] = np.arange(p0, p0 + B)"),
 ("lse in log2", "lse = (m + np.log(l))[:, 0]", "lse = (m + np.log2(l))[:, 0]"),
 ("top-k takes the lowest scores", "order = np.lexsort((j, -s))", "order = np.lexsort((j, s))"),
 ("key-block bwd: Delta dropped", "Dq = (do * o).sum(axis=1, keepdims=True)          # = sum_k", "Dq = 0.0 * (do * o).sum(axis=1, keepdims=True)  # = sum_k"),
 ("key-block bwd: dK without scale", "dK += scale * (dSj.T @ q)", "dK += dSj.T @ q"),
 ("key-block bwd: wrong column offset", "at = int(np.searchsorted(np.asarray(ids), j))", "at = int(np.searchsorted(np.asarray(ids), j)) + 0 * len(ids) - (1 if j > 0 else 0)"),
 ("key-block bwd: dV from dS", "dV += Pj.T @ do", "dV += dSj.T @ do"),
]


BENCH = [
 ("pairs: wrong head offset", "Bk = Bsz[head_of * NB + col]", "Bk = Bsz[col]"),
 ("pairs: query size from the key", "return int((Bq[row_of] * Bk).sum().item())", "return int((Bk * Bk).sum().item())"),
 ("roofline: work not scaled by steps", "per_launch = work * steps / n", "per_launch = work / n"),
 ("roofline: fp32 peak counts FMA twice", "rec[\"peak\"] = 148 * 128 * peaks", "rec[\"peak\"] = 148 * 256 * peaks"),
 ("roofline: fwd work 2PD", "\"attn_fwd\": (\"tensor\", 4.0 * P * D,", "\"attn_fwd\": (\"tensor\", 2.0 * P * D,"),
 ("whole-job rate of one rank", "return world * units_per_rank / (ms_max * 1e-3)", "return units_per_rank / (ms_max * 1e-3)"),
 ("head ranges ignore the remainder", "h0 = rank * base + min(rank, extra)", "h0 = rank * base"),
 ("max over ranks sums", "torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)", "torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)"),
 ("sample: row fraction inverted", "row_frac = nb / len(sel_rows)", "row_frac = len(sel_rows) / nb"),
 ("sample: pairs not scaled to the heads", "P_total = pairs_rows * row_frac * w.heads", "P_total = pairs_rows * row_frac"),
 ("selection share over 2N", "\"key_share_per_row\": summary(keys[valid] / N)}", "\"key_share_per_row\": summary(keys[valid] / (2 * N))}"),
 ("selection counts every row", "\"blocks_per_row\": summary(counts[valid].double())", "\"blocks_per_row\": summary(counts.double())"),
 ("digest keeps comments", "            i = n if j < 0 else j\n", "            out.append(text[i:n if j < 0 else j])\n            i = n if j < 0 else j\n"),
 ("digest ignores includes", "            todo.append(os.path.normpath(os.path.join(os.path.dirname(path), inc)))", "            pass"),
 ("stale traffic still reported", "        if source_digest(d[\"source\"]) != d[\"code_digest\"]:", "        if False:"),
 ("clock median as mean", "return {\"sm_mhz\": statistics.median(sm) if sm else None", "return {\"sm_mhz\": statistics.mean(sm) if sm else None"),
 ("throttle reasons ignored", "                if v.strip().lower() == \"active\":", "                if False:"),
 ("fused backward issued as 14PD", "\"issued_TFLOPs\": (10.0 if one else 14.0)", "\"issued_TFLOPs\": (14.0 if one else 14.0)"),
 ("accumulator zeroing not counted", "(12.0 if fused else 8.0) * HBD", "8.0 * HBD"),
 ("e2e: a step does not wait for its inputs", "            cs.wait_event(ev_in[b])\n", "            pass\n"),
 ("e2e: results copied before the step ends", "            xs.wait_event(ev_done[b])\n            with torch.cuda.stream(xs):\n                for src, dst",
  "            with torch.cuda.stream(xs):\n                for src, dst"),
]

BINDING = [
 ("binding: shape unchecked", "    if tuple(t.shape) != tuple(shape):\n        raise", "    if False:\n        raise"),
 ("binding: dtype unchecked", "    if t.dtype != dtype:\n        raise", "    if False:\n        raise"),
 ("binding: grid unchecked", "    if _grid(p) != _grid(q):", "    if False:"),
 ("binding: host tensors accepted", "        if not t.is_cuda:\n            raise", "        if False:\n            raise"),
 ("binding: capacity unchecked", "    if not 0 <= sel.nnz <= cap:", "    if False:"),
 ("binding: transpose not required", "    elif transpose:\n        raise", "    elif False:\n        raise"),
 ("binding: caller's stream ignored", "    s = stream if stream is not None else torch.cuda.current_stream(device)",
  "    s = torch.cuda.current_stream(device)"),
 ("binding: no growth on short capacity", "out.col.numel() < cs.nnz <= 0x7fffffff", "False"),
 ("binding: residual always passed", "_ptr(O_res) if residual else None, _ptr(lse)", "_ptr(O_res), _ptr(lse)"),
 ("binding: gradients in the wrong order", "_ptr(dQ), _ptr(dK), _ptr(dV)", "_ptr(dK), _ptr(dQ), _ptr(dV)"),
 ("binding: backward path selector dropped", "int(bool(deterministic))", "0"),
]

CABI = [  # (file under the package's csrc/, name, old, new); the copy's library is rebuilt for each
 ("api.cu", "C: backward path selector unchecked", "if (deterministic != 0 && deterministic != 1)", "if (false)"),
 ("api.cu", "C: zone edge unchecked", "if (p->T % 8 || p->H % 8 || p->W % 8)", "if (false)"),
 ("api.cu", "C: head_dim 96 accepted", "if (p->head_dim != 64 && p->head_dim != 128)", "if (false)"),
 ("api.cu", "C: grid size unchecked", "if (N * p->heads * p->head_dim >= (1LL << 40) || N >= (1LL << 30))", "if (false)"),
 ("api.cu", "C: thresholds unchecked", "if (!(p->tau128 >= p->tau256) || !(p->tau256 >= 0.f) || !isfinite(p->tau128))", "if (false)"),
 ("api.cu", "C: eps unchecked", "if (!(p->eps > 0.f) || !isfinite(p->eps))", "if (false)"),
 ("api.cu", "C: top_p unchecked", "if (!(p->top_p >= 0.f) || !isfinite(p->top_p))", "if (false)"),
 ("api.cu", "C: top-k unchecked", "if (p->topk_abs < 0 || !(p->topk_frac >= 0.f) || !isfinite(p->topk_frac))", "if (false)"),
 ("api.cu", "C: sm_scale unchecked", "if (p->sm_scale < 0.f || !isfinite(p->sm_scale))", "if (false)"),
 ("api.cu", "C: map_exponent unchecked", "if (!(p->map_exponent >= 0.f && p->map_exponent <= 8.f))", "if (false)"),
 ("api.cu", "C: guidance unchecked", "if (p->guidance < 0 || p->guidance > 3)", "if (false)"),
 ("api.cu", "C: density unchecked", "if (p->density < 0 || p->density > 3)", "if (false)"),
 ("api.cu", "C: alignment unchecked", "if (reinterpret_cast<uintptr_t>(ptr) % 16) return fail(", "if (false) return fail("),
 ("api.cu", "C: workspace size unchecked", "if (bytes < need) return fail(", "if (false) return fail("),
 ("api.cu", "C: workspace alignment unchecked", "if (reinterpret_cast<uintptr_t>(ws) % 256)", "if (false)"),
 ("api.cu", "C: density 3 without norms", "if (p->density == 3 && !a2v_norm)", "if (false)"),
 ("api.cu", "C: backward without transpose", "if (!sel || !sel->row_ptr || !sel->col || !sel->col_ptr || !sel->row)", "if (!sel || !sel->row_ptr || !sel->col)"),
 ("a2v_norm.cu", "C: a2v width not a multiple of 8", "if (width <= 0 || width % 8 || width > (1 << 20))", "if (width <= 0 || width > (1 << 20))"),
 ("a2v_norm.cu", "C: a2v ld below width", "if (ld < width || ld % 8)", "if (ld % 8)"),
 ("a2v_norm.cu", "C: a2v negative n", "if (n < 0) return", "if (false) return"),
 ("timing.cu", "C: timing id unchecked", "if (id < 0 || id >= KT_COUNT) return", "if (false) return"),
]

def main(only):
    tmp = tempfile.mkdtemp(prefix="mutation_check_")
    dst = os.path.join(tmp, "repo")
    try:
        # the copy holds the tracked files only (the committed repository)
        tracked = subprocess.run(["git", "ls-files", "-z"], cwd=ROOT, capture_output=True, check=True).stdout
        for rel in tracked.decode().split("\0"):
            if rel:
                os.makedirs(os.path.dirname(os.path.join(dst, rel)), exist_ok=True)
                shutil.copy2(os.path.join(ROOT, rel), os.path.join(dst, rel))
        subprocess.run([sys.executable, "-m", "dynamic_block_sparse_stats_b200.build", "--force"], cwd=dst,
                       capture_output=True, check=True)
        survivors = []
        for target, entries in (("oracle/prism_oracle.py", M), ("bench.py", BENCH),
                                 ("dynamic_block_sparse_stats_b200/api.py", BINDING)):
            path = os.path.join(dst, target)
            with open(path) as f:
                orig = f.read()
            for name, old, new in entries:
                if only and name not in only:
                    continue
                if orig.count(old) != 1:
                    print(f"SKIP     {name}: pattern found {orig.count(old)} times in {target}")
                    continue
                with open(path, "w") as f:
                    f.write(orig.replace(old, new))
                t = time.time()
                r = subprocess.run([sys.executable, "-m", "pytest", "tests", "-x", "-q", "-m", "not gpu",
                                    "-p", "no:cacheprovider", "--deselect",
                                    "tests/test_bench_reference_cpu.py::"
                                    "test_reference_arm_under_torchrun_prints_one_line_from_rank_zero"],
                                   cwd=dst, capture_output=True, text=True)
                failed = [ln for ln in r.stdout.splitlines() if ln.startswith(("FAILED", "ERROR"))][:1]
                if r.returncode == 0:
                    survivors.append(name)
                print(f"{'caught  ' if r.returncode else 'SURVIVED'} {name:38s} {time.time() - t:5.1f}s {failed}",
                      flush=True)
            with open(path, "w") as f:
                f.write(orig)
        csrc = os.path.join(dst, "dynamic_block_sparse_stats_b200", "csrc")
        build = [sys.executable, "-m", "dynamic_block_sparse_stats_b200.build", "--force"]
        for fname, name, old, new in CABI:
            if only and name not in only:
                continue
            path = os.path.join(csrc, fname)
            with open(path) as f:
                orig = f.read()
            if orig.count(old) != 1:
                print(f"SKIP     {name}: pattern found {orig.count(old)} times in {fname}")
                continue
            with open(path, "w") as f:
                f.write(orig.replace(old, new))
            t = time.time()
            b = subprocess.run(build, cwd=dst, capture_output=True, text=True)
            if b.returncode != 0:
                print(f"NOBUILD  {name}")
            else:
                r = subprocess.run([sys.executable, "-m", "pytest", "tests", "-x", "-q", "-m", "not gpu",
                                    "-p", "no:cacheprovider", "--deselect",
                                    "tests/test_bench_reference_cpu.py::"
                                    "test_reference_arm_under_torchrun_prints_one_line_from_rank_zero"],
                                   cwd=dst, capture_output=True, text=True)
                failed = [ln for ln in r.stdout.splitlines() if ln.startswith(("FAILED", "ERROR"))][:1]
                if r.returncode == 0:
                    survivors.append(name)
                print(f"{'caught  ' if r.returncode else 'SURVIVED'} {name:38s} {time.time() - t:5.1f}s {failed}",
                      flush=True)
            with open(path, "w") as f:
                f.write(orig)
            subprocess.run(build, cwd=dst, capture_output=True, text=True)
        print("survivors:", survivors)
        return 1 if survivors else 0
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
