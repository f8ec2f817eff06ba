// CUDA-graph replay of the block decode (kda_block_decode_graph): a serving loop that decodes
// the same N sequences from the same buffers every step records the call's kernels once and
// replays them with one launch, so the per-step cost is the kernels alone, not the host's
// launch of each of them (Glm5NextLayer's CUDA-graph hooks, at the level of one block).
#include "common.cuh"

struct kda_graph {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
};

extern "C" int kda_block_decode_graph(const kda_block_weights *w, const kda_bf16 *hidden, int N,
                                      float *const *h_state, kda_bf16 *const *conv_state, kda_workspace *ws,
                                      kda_graph **out) {
    if (!out) return KDA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!w || !hidden || !h_state || !conv_state || !ws || N < 1) return KDA_ERR_INVALID_ARG;
    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return KDA_ERR_CUDA;
    // relaxed: the call's one-time attribute and symbol look-ups are not stream work
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
        cudaStreamDestroy(cs);
        return KDA_ERR_CUDA;
    }
    const int rc = kda_block_decode(w, hidden, N, h_state, conv_state, ws, cs);
    cudaGraph_t g = nullptr;
    const cudaError_t e = cudaStreamEndCapture(cs, &g);
    cudaStreamDestroy(cs);
    if (rc != KDA_OK || e != cudaSuccess || !g) {
        if (g) cudaGraphDestroy(g);
        cudaGetLastError();  // a failed capture leaves no sticky error behind
        return rc != KDA_OK ? rc : KDA_ERR_CUDA;
    }
    cudaGraphExec_t x = nullptr;
    if (cudaGraphInstantiate(&x, g, 0) != cudaSuccess) {
        cudaGraphDestroy(g);
        return KDA_ERR_CUDA;
    }
    *out = new kda_graph{g, x};
    return KDA_OK;
}

extern "C" int kda_graph_launch(kda_graph *g, void *stream) {
    if (!g) return KDA_ERR_INVALID_ARG;
    return cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" int kda_graph_destroy(kda_graph *g) {
    if (!g) return KDA_OK;
    cudaGraphExecDestroy(g->exec);
    cudaGraphDestroy(g->graph);
    delete g;
    return KDA_OK;
}
