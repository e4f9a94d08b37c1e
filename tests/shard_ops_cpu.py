"""A CPU stand-in for the per-rank steps of vocabulary-sharded verification
(the spec_shard_* kernels), with the same inputs, outputs and layouts, in
plain fp64 numpy.  Test infrastructure only: it lets the multi-rank protocol
of speculative_decoding_verification_87_b200.sharded run over gloo on CPU
processes.  The kernels themselves are checked on the GPU against the
oracle; this module checks only that the protocol (what is exchanged, in
which order, which rank draws) reproduces the single-rank result.  Random
numbers come from the oracle's Philox."""
import numpy as np
import torch

import oracle

MODE_NONE, MODE_TARGET, MODE_RESIDUAL = 0, 1, 2
INT_MAX = 2 ** 31 - 1


def _f64(t, ncols):
    """CPU logits (fp32 or bf16 tensor) -> fp64 numpy of the first ncols columns."""
    return t[..., :ncols].to(torch.float64).numpy()


def _accept(lp, lq, u):
    if lp == -np.inf:
        return False
    if lq == -np.inf or lp >= lq:
        return True
    if u == 0.0:
        return True
    return np.log(u) + lq < lp


class CpuShardOps:
    def row_stats(self, target, draft, tokens, lo, hi, temperature):
        n = hi - lo
        rows = [_f64(target, n)]
        if draft is not None:
            rows.append(_f64(draft, n))
        x = np.concatenate(rows, axis=1)  # [B][R][n]
        B, R, _ = x.shape
        mx = np.full((B, R), -np.inf)
        arg = np.full((B, R), INT_MAX, np.int64)
        sm = np.zeros((B, R))
        for b in range(B):
            for r in range(R):
                row = x[b, r]
                if np.isnan(row).any():
                    mx[b, r] = np.nan
                    sm[b, r] = np.nan
                    continue
                m = row.max()
                mx[b, r] = m
                if m != -np.inf:
                    arg[b, r] = lo + int(np.argmax(row == m))
                    sm[b, r] = np.exp((row[row != -np.inf] - m) / temperature).sum()
        out = dict(max=torch.from_numpy(mx.astype(np.float32)))
        if draft is None:
            out["arg"] = torch.from_numpy(arg.astype(np.int32))
            return out
        out["sum"] = torch.from_numpy(sm)
        k = tokens.shape[1]
        tk = tokens.numpy()
        probe = np.full((B, k, 2), np.nan, np.float32)
        t64, d64 = _f64(target, n), _f64(draft, n)
        for b in range(B):
            for j in range(k):
                if lo <= tk[b, j] < hi:
                    probe[b, j] = (t64[b, j, tk[b, j] - lo], d64[b, j, tk[b, j] - lo])
        out["probe"] = torch.from_numpy(probe)
        return out

    def decide(self, max_all, sum_all, probe_all, bounds, tokens, vocab, temperature, seed, offset,
               status):
        mx, sm, pr = max_all.numpy().astype(np.float64), sum_all.numpy(), probe_all.numpy()
        bd = bounds.numpy()
        W, B, R = mx.shape
        k = (R - 1) // 2
        tk = tokens.numpy()
        ua = oracle.uniforms(seed, offset, oracle.ACCEPT, B, k)
        us = oracle.uniforms(seed, offset, oracle.SAMPLE, B, k + 1)
        out = np.full((B, k + 1), -1, np.int32)
        acc = np.zeros(B, np.int32)
        draw = np.zeros((B, 6))
        bits_all = 0
        for b in range(B):
            M = np.empty(R)
            S = np.empty(R)
            for r in range(R):
                col = mx[:, b, r]
                if np.isnan(col).any() or np.isnan(sm[:, b, r]).any():
                    M[r] = S[r] = np.nan
                    continue
                M[r] = col.max()
                S[r] = sum(sm[w, b, r] * np.exp((col[w] - M[r]) / temperature)
                           for w in range(W) if col[w] != -np.inf) if M[r] != -np.inf else 0.0
            bad = not all(np.isfinite(M[r]) and np.isfinite(S[r]) and S[r] > 0 for r in range(R))
            tok_bad = any(not 0 <= tk[b, j] < vocab for j in range(k))
            bits = (1 if tok_bad else 0) | (4 if bad else 0)
            if bits:
                bits_all |= bits
                acc[b] = -1
                continue
            n = k
            for j in range(k):
                w = int(np.searchsorted(bd, tk[b, j], side="right")) - 1
                lt, ld = pr[w, b, j]
                lp = (lt - M[j]) / temperature - np.log(S[j])
                lq = (ld - M[k + 1 + j]) / temperature - np.log(S[k + 1 + j])
                if not _accept(lp, lq, ua[b, j]):
                    n = j
                    break
            out[b, :n] = tk[b, :n]
            acc[b] = n
            draw[b] = (MODE_RESIDUAL if n < k else MODE_TARGET, n, M[n],
                       M[k + 1 + n] if n < k else 0.0, us[b, n], 0.0)
        if status is not None and bits_all:
            status |= bits_all
        return torch.from_numpy(out), torch.from_numpy(acc), torch.from_numpy(draw)

    def decide_greedy(self, max_all, arg_all, tokens, vocab, status):
        mx, ag = max_all.numpy(), arg_all.numpy()
        W, B, R = mx.shape
        k = R - 1
        tk = tokens.numpy()
        out = np.full((B, k + 1), -1, np.int32)
        acc = np.zeros(B, np.int32)
        bits_all = 0
        for b in range(B):
            g = []
            nan = False
            for r in range(R):
                best, bi = -np.inf, INT_MAX
                for w in range(W):
                    v = mx[w, b, r]
                    if np.isnan(v):
                        nan = True
                    elif v > best or (v == best and ag[w, b, r] < bi):
                        best, bi = v, ag[w, b, r]
                g.append(0 if bi == INT_MAX else int(bi))
            tok_bad = any(not 0 <= tk[b, j] < vocab for j in range(k))
            bits = (1 if tok_bad else 0) | (4 if nan else 0)
            if bits:
                bits_all |= bits
                acc[b] = -1
                continue
            n = next((j for j in range(k) if tk[b, j] != g[j]), k)
            out[b, :n] = tk[b, :n]
            out[b, n] = g[n]
            acc[b] = n
        if status is not None and bits_all:
            status |= bits_all
        return torch.from_numpy(out), torch.from_numpy(acc)

    @staticmethod
    def _weights(target, draft, lo, hi, temperature, d, b, isp=None, isq=None, residual=None):
        n = hi - lo
        j = int(d[1])
        e = np.exp((_f64(target[b, j], n) - d[2]) / temperature)
        if d[0] == MODE_RESIDUAL:
            f = np.exp((_f64(draft[b, j], n) - d[3]) / temperature)
        else:
            f = np.zeros_like(e)
        if isp is None:
            return e, f
        if residual:
            return np.maximum(e * isp - f * isq, 0.0), e
        return e, e

    def draw_sums(self, target, draft, lo, hi, temperature, draw, norm_parts):
        dr = draw.numpy()
        B = dr.shape[0]
        sums = np.zeros((B, 2))
        for b in range(B):
            d = dr[b]
            if d[0] == MODE_NONE:
                continue
            if norm_parts is None:
                e, f = self._weights(target, draft, lo, hi, temperature, d, b)
                sums[b] = (e.sum(), f.sum())
            else:
                npr = norm_parts.numpy()
                St = sum(npr[w, b, 0] for w in range(npr.shape[0]))
                Sd = sum(npr[w, b, 1] for w in range(npr.shape[0]))
                res = d[0] == MODE_RESIDUAL
                w, e = self._weights(target, draft, lo, hi, temperature, d, b, 1 / St,
                                     (1 / Sd) if res else 0.0, res)
                sums[b] = (w.sum(), e.sum())
        return torch.from_numpy(sums)

    def draw_pick(self, target, draft, lo, hi, temperature, draw, norm_parts, mass_parts, me):
        dr, npr, mp = draw.numpy(), norm_parts.numpy(), mass_parts.numpy()
        W = npr.shape[0]
        B = dr.shape[0]
        token = np.full(B, -1, np.int32)
        for b in range(B):
            d = dr[b]
            if d[0] == MODE_NONE:
                continue
            res = d[0] == MODE_RESIDUAL
            which = 0
            Z = sum(mp[w, b, 0] for w in range(W))
            if res and not Z > 0:
                which, res = 1, False
                Z = sum(mp[w, b, 1] for w in range(W))
            target_u = d[4] * Z
            run, owner, before, last, last_before = 0.0, -1, 0.0, -1, 0.0
            for w in range(W):
                m = mp[w, b, which]
                if m > 0:
                    if run + m > target_u:
                        owner, before = w, run
                        break
                    last, last_before = w, run
                run += m
            if owner < 0:
                owner, before = last, last_before
            if owner != me:
                continue
            St = sum(npr[w, b, 0] for w in range(W))
            Sd = sum(npr[w, b, 1] for w in range(W))
            wts, _ = self._weights(target, draft, lo, hi, temperature, d, b, 1 / St,
                                   (1 / Sd) if res else 0.0, res)
            c = np.cumsum(wts)
            t = target_u - before
            hit = np.nonzero((wts > 0) & (c > t))[0]
            v = int(hit[0]) if len(hit) else int(np.nonzero(wts > 0)[0][-1])
            token[b] = lo + v
        return torch.from_numpy(token)

    def emit(self, token, draw, out):
        dr = draw.numpy()
        for b in range(dr.shape[0]):
            if dr[b, 0] != MODE_NONE:
                out[b, int(dr[b, 1])] = int(token[b])
