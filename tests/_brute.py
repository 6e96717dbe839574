"""Brute-force, scalar-loop restatement of the streaming step for tiny inputs.

Written independently of the oracle (no numpy matmul, no shared helpers): every
projection is an explicit sum, RoPE is an explicit 2x2 rotation per pair with
math.cos / math.sin, attention loops over keys and decides visibility from the
block rule, and the schedule uses the closed form "at tick k slot i runs block
k - i".  Used only to pin the oracle on tiny configs.
"""
import math


def matvec_rows(X, W):
    """Y[t][n] = sum_k X[t][k] * W[n][k] (W in [out, in] layout)."""
    out = []
    for row in X:
        out.append([sum(row[k] * wn[k] for k in range(len(row))) for wn in W])
    return out


def normalize_rows(X, eps=1e-6):
    """Each row divided by the square root of (its mean square + eps)."""
    out = []
    for row in X:
        ms = sum(v * v for v in row) / len(row)
        s = math.sqrt(ms + eps)
        out.append([v / s for v in row])
    return out


def rotate(vec, t, r, c, pairs, theta):
    pt, ph, pw = pairs
    res = list(vec)
    for j in range(len(vec) // 2):
        if j < pt:
            ang = t * theta ** (-(j) / pt)
        elif j < pt + ph:
            ang = r * theta ** (-(j - pt) / ph)
        else:
            ang = c * theta ** (-(j - pt - ph) / pw)
        a, b = vec[2 * j], vec[2 * j + 1]
        res[2 * j] = a * math.cos(ang) - b * math.sin(ang)
        res[2 * j + 1] = a * math.sin(ang) + b * math.cos(ang)
    return res


class BruteStream:
    def __init__(self, cfg, W):
        self.c = cfg
        tolist = lambda a: None if a is None else [[float(v) for v in row] for row in a]
        self.wqkv = [tolist(w) for w in W.w_qkv]
        self.wout = [tolist(w) for w in W.w_out]
        self.win = tolist(W.w_in)
        self.whead = tolist(W.w_head)
        self.keys = []        # entries (layer, slot, block, token_pos, k_vec_per_head, v_vec_per_head)
        self.sink = None      # per layer: list of (r, c, k_heads (unroped), v_heads)
        self.replaced = False
        self.lat = {}
        self.clean = []       # clean-cache entries (layer, block, k_rot, v)
        self.dit = getattr(cfg, "block_kind", 0) == 1
        if self.dit:
            self.w1 = [tolist(w) for w in W.w_ffn1]
            self.w2 = [tolist(w) for w in W.w_ffn2]
            self.ada = [[[[float(v) for v in vec] for vec in st] for st in lay] for lay in W.ada]
        self.cross = self.dit and getattr(cfg, "audio_tokens", 0) > 0
        if self.cross:
            self.wqc = [tolist(w) for w in W.w_qc]
            self.wkvc = [tolist(w) for w in W.w_kvc]
            self.woc = [tolist(w) for w in W.w_oc]
        self.audio = {}

    # -- the DiT block's pieces, scalar ------------------------------------------------------------
    def _operand(self, h, l, t_idx):
        """Per-token RMS norm, AdaLN-modulated in the DiT block."""
        n = normalize_rows(h)
        if not self.dit:
            return n
        sh, sc = self.ada[l][t_idx][0], self.ada[l][t_idx][1]
        return [[v * (1.0 + sc[j]) + sh[j] for j, v in enumerate(row)] for row in n]

    def _cross(self, h, l, audio):
        """The audio cross-attention sub-block's contribution, scalar."""
        c = self.c
        D = c.hidden
        q = matvec_rows(normalize_rows(h), self.wqc[l])
        kv = matvec_rows([list(map(float, r)) for r in audio], self.wkvc[l])
        qh = [[row[hh * c.head_dim:(hh + 1) * c.head_dim] for hh in range(c.heads)] for row in q]
        keys = [([row[hh * c.head_dim:(hh + 1) * c.head_dim] for hh in range(c.heads)],
                 [row[D + hh * c.head_dim:D + (hh + 1) * c.head_dim] for hh in range(c.heads)]) for row in kv]
        return matvec_rows(self._layer_attend(qh, keys), self.woc[l])

    def _residual(self, h, proj, l, t_idx, audio=None):
        """h + attention output; in the DiT block gated, then + the audio cross-attention
        (when the block has audio), then + gated tanh-GELU FFN."""
        if not self.dit:
            return [[a + b for a, b in zip(hr, pr)] for hr, pr in zip(h, proj)]
        a = self.ada[l][t_idx]
        h = [[x + a[2][j] * p for j, (x, p) in enumerate(zip(hr, pr))] for hr, pr in zip(h, proj)]
        if audio is not None:
            cr = self._cross(h, l, audio)
            h = [[x + y for x, y in zip(hr, cr_)] for hr, cr_ in zip(h, cr)]
        n = normalize_rows(h)
        m = [[v * (1.0 + a[4][j]) + a[3][j] for j, v in enumerate(row)] for row in n]
        u = matvec_rows(m, self.w1[l])
        g = [[0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z * z * z))) for z in row]
             for row in u]
        f = matvec_rows(g, self.w2[l])
        return [[x + a[5][j] * y for j, (x, y) in enumerate(zip(hr, fr))] for hr, fr in zip(h, f)]

    def _heads(self, vec, part):
        c = self.c
        D, d = c.hidden, c.head_dim
        return [vec[part * D + h * d: part * D + (h + 1) * d] for h in range(c.heads)]

    def _tok_rc(self, n):
        F, gw = self.c.frame_tokens, self.c.grid_w
        f, rem = divmod(n, F)
        return f, rem // gw, rem % gw

    def _layer_attend(self, qs_heads, key_list):
        """qs_heads: per query, per head rotated q; key_list: [(k_heads, v_heads)]."""
        c = self.c
        outs = []
        for qh in qs_heads:
            row = []
            for h in range(c.heads):
                logits = [sum(qh[h][e] * kh[h][e] for e in range(c.head_dim)) / math.sqrt(c.head_dim)
                          for kh, _ in key_list]
                mx = max(logits)
                ws = [math.exp(z - mx) for z in logits]
                tot = sum(ws)
                acc = [0.0] * c.head_dim
                for wgt, (_, vh) in zip(ws, key_list):
                    for e in range(c.head_dim):
                        acc[e] += wgt / tot * vh[h][e]
                row.extend(acc)
            outs.append(row)
        return outs

    def set_sink(self, latent):
        c = self.c
        h = [list(map(float, r)) for r in latent]
        if self.win is not None:
            h = matvec_rows(h, self.win)
        t0 = -c.sink_offset_frames
        self.sink = []
        for l in range(c.num_layers):
            qkv = matvec_rows(self._operand(h, l, c.num_steps), self.wqkv[l])
            entries, qrot, krot = [], [], []
            for n, vec in enumerate(qkv):
                _, r, cc = self._tok_rc(n)
                qh, kh, vh = self._heads(vec, 0), self._heads(vec, 1), self._heads(vec, 2)
                entries.append((r, cc, kh, vh))
                qrot.append([rotate(x, t0, r, cc, c.pairs, c.rope_theta) for x in qh])
                krot.append(([rotate(x, t0, r, cc, c.pairs, c.rope_theta) for x in kh], vh))
            self.sink.append(entries)
            o = self._layer_attend(qrot, krot)
            proj = matvec_rows(o, self.wout[l])
            h = self._residual(h, proj, l, c.num_steps)

    def step(self, x, b, i, win_step=None):
        """Block b at step i; the prior blocks' K/V come from step win_step's entries
        (default: step i's own, timestep forcing)."""
        c = self.c
        ws = i if win_step is None else win_step
        h = [list(map(float, r)) for r in x]
        if self.win is not None:
            h = matvec_rows(h, self.win)
        fpb = c.frames_per_block
        t_sink = fpb * b - c.sink_offset_frames if c.rolling_rope else -c.sink_offset_frames
        for l in range(c.num_layers):
            qkv = matvec_rows(self._operand(h, l, i), self.wqkv[l])
            qrot = []
            for n, vec in enumerate(qkv):
                f, r, cc = self._tok_rc(n)
                t = fpb * b + f
                qrot.append([rotate(x_, t, r, cc, c.pairs, c.rope_theta) for x_ in self._heads(vec, 0)])
                kr = [rotate(x_, t, r, cc, c.pairs, c.rope_theta) for x_ in self._heads(vec, 1)]
                self.keys.append((l, i, b, kr, self._heads(vec, 2)))
            visible = []
            for (r, cc, kh, vh) in self.sink[l]:
                visible.append(([rotate(x_, t_sink, r, cc, c.pairs, c.rope_theta) for x_ in kh], vh))
            for (ll, ii, bb, kr, vh) in self.keys:
                if ll == l and ((ii == ws and b - c.window_blocks <= bb < b) or (ii == i and bb == b)):
                    visible.append((kr, vh))
            o = self._layer_attend(qrot, visible)
            proj = matvec_rows(o, self.wout[l])
            h = self._residual(h, proj, l, i, self.audio.get(b) if self.cross else None)
        hn = normalize_rows(h)
        v = hn if self.whead is None else matvec_rows(hn, self.whead)
        dt = c.timesteps[i + 1] - c.timesteps[i]
        return [[xa + dt * va for xa, va in zip(xr, vr)] for xr, vr in zip(x, v)]

    def run_sequential_fixed(self, noises, win_step):
        """Each block through its num_steps Euler steps in order; every step reads the
        prior blocks' K/V written at step win_step (the fixed-noise cache)."""
        c = self.c
        done = {}
        for b, nz in enumerate(noises):
            x = [list(map(float, r)) for r in nz]
            for i in range(c.num_steps):
                x = self.step(x, b, i, win_step=win_step)
            done[b] = x
            if b == 0 and c.sink_mode == 1 and not self.replaced:
                self.replaced = True
                self.set_sink(x[: c.sink_tokens])
        return done

    def run_pipelined(self, noises, audios=None):
        """Tick k: slot i runs block k - i.  Returns {block: final latent}."""
        c = self.c
        if audios is not None:
            self.audio = dict(enumerate(audios))
        S = c.num_steps
        nb = len(noises)
        done = {}
        for k in range(nb + S - 1):
            for i in range(S):
                b = k - i
                if 0 <= b < nb:
                    x = self.lat.get(b, [list(map(float, r)) for r in noises[b]]) if i == 0 else self.lat[b]
                    self.lat[b] = self.step(x, b, i)
            fin = k - (S - 1)
            if 0 <= fin < nb:
                done[fin] = self.lat.pop(fin)
                if fin == 0 and c.sink_mode == 1 and not self.replaced:
                    self.replaced = True
                    self.set_sink(done[0][: c.sink_tokens])
        return done

    # -- clean-cache refresh (NFE num_steps + 1), sequential -------------------------
    def _forward_clean(self, x, b):
        """One pass of block b over the clean cache: every layer attends to the
        sink, the clean K/V of blocks b - window .. b - 1 and the pass's own K/V.
        Returns (final residual, [(layer, [(k_rot, v) per token])])."""
        c = self.c
        h = [list(map(float, r)) for r in x]
        if self.win is not None:
            h = matvec_rows(h, self.win)
        fpb = c.frames_per_block
        t_sink = fpb * b - c.sink_offset_frames if c.rolling_rope else -c.sink_offset_frames
        own_all = []
        for l in range(c.num_layers):
            qkv = matvec_rows(normalize_rows(h), self.wqkv[l])
            qrot, own = [], []
            for n, vec in enumerate(qkv):
                f, r, cc = self._tok_rc(n)
                t = fpb * b + f
                qrot.append([rotate(x_, t, r, cc, c.pairs, c.rope_theta) for x_ in self._heads(vec, 0)])
                own.append(([rotate(x_, t, r, cc, c.pairs, c.rope_theta) for x_ in self._heads(vec, 1)],
                            self._heads(vec, 2)))
            visible = [([rotate(x_, t_sink, r, cc, c.pairs, c.rope_theta) for x_ in kh], vh)
                       for (r, cc, kh, vh) in self.sink[l]]
            visible += [(kr, vh) for (ll, bb, kr, vh) in self.clean if ll == l and b - c.window_blocks <= bb < b]
            visible += own
            o = self._layer_attend(qrot, visible)
            proj = matvec_rows(o, self.wout[l])
            h = [[a + bq for a, bq in zip(hr, pr)] for hr, pr in zip(h, proj)]
            own_all.append((l, own))
        return h, own_all

    def run_sequential_clean(self, noises):
        """Each block: num_steps Euler steps over the clean cache, then one more
        pass of the finished latent whose K/V become that block's clean entry."""
        c = self.c
        self.clean = []       # (layer, block, k_rot, v)
        done = {}
        for b, noise in enumerate(noises):
            x = [list(map(float, r)) for r in noise]
            for i in range(c.num_steps):
                h, _ = self._forward_clean(x, b)
                hn = normalize_rows(h)
                v = hn if self.whead is None else matvec_rows(hn, self.whead)
                dt = c.timesteps[i + 1] - c.timesteps[i]
                x = [[xa + dt * va for xa, va in zip(xr, vr)] for xr, vr in zip(x, v)]
            _, own_all = self._forward_clean(x, b)
            for l, own in own_all:
                for kr, vh in own:
                    self.clean.append((l, b, kr, vh))
            done[b] = x
            if b == 0 and c.sink_mode == 1 and not self.replaced:
                self.replaced = True
                self.set_sink(x[: c.sink_tokens])
        return done
