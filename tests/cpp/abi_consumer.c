/*
 * A plain C99 consumer of libllama_b200.so: it includes both public headers,
 * links the shared library, and calls the entry points that do their work on
 * the host (configuration sizing, argument checks, the error message, the
 * launch counter).  It proves that the headers are valid C and that the
 * exported symbols, struct layouts and status codes are usable from C
 * without any C++ or Python in between.  It launches no kernel and needs no
 * GPU.
 *
 * Output, one record per line (parsed by tests/test_abi_c_consumer.py):
 *   sizes <sizeof args> <sizeof sampling>
 *   bytes <name> <rc> <weights> <kv> <workspace> <total> <hidden>
 *   check <what> <rc> <llama_last_error() after the call>
 *   launches <count>
 *   done
 */
#include <stdio.h>
#include <string.h>

#include "llama_b200.h"
#include "llama_b200_ops.h"

static llama_model_args shape(int dim, int n_layers, int n_heads, int n_kv_heads, int vocab, int multiple_of,
                              float mult, int max_seq_len, int max_batch, int dtype) {
    llama_model_args a;
    memset(&a, 0, sizeof(a));
    a.dim = dim;
    a.n_layers = n_layers;
    a.n_heads = n_heads;
    a.n_kv_heads = n_kv_heads;
    a.vocab_size = vocab;
    a.multiple_of = multiple_of;
    a.ffn_dim_multiplier = mult;
    a.norm_eps = 1e-5f;
    a.rope_theta = 10000.0f;
    a.max_seq_len = max_seq_len;
    a.max_batch_size = max_batch;
    a.max_tokens = 0;
    a.dtype = dtype;
    return a;
}

static void bytes_line(const char* name, const llama_model_args* a) {
    size_t w = 0, kv = 0, ws = 0, total = 0;
    int32_t hidden = 0;
    const int rc = llama_model_bytes(a, &w, &kv, &ws, &total, &hidden);
    printf("bytes %s %d %zu %zu %zu %zu %d\n", name, rc, w, kv, ws, total, (int)hidden);
}

static void check_line(const char* what, int rc) {
    const char* msg = llama_last_error();
    printf("check %s %d %s\n", what, rc, msg != NULL ? msg : "");
}

int main(void) {
    printf("sizes %zu %zu\n", sizeof(llama_model_args), sizeof(llama_sampling));

    /* Llama-2 7B, 13B and the 70B layer shape (grouped-query attention, 8 KV
     * heads, ffn_dim_multiplier 1.3 and multiple_of 4096), and a tiny model. */
    llama_model_args a7 = shape(4096, 32, 32, 32, 32000, 256, 0.0f, 4096, 4, LLAMA_BF16);
    llama_model_args a13 = shape(5120, 40, 40, 40, 32000, 256, 0.0f, 1152, 16, LLAMA_F16);
    llama_model_args a70 = shape(8192, 16, 64, 8, 32000, 4096, 1.3f, 4096, 8, LLAMA_BF16);
    llama_model_args tiny = shape(256, 2, 8, 2, 512, 256, 0.0f, 128, 2, LLAMA_F32);
    bytes_line("7b", &a7);
    bytes_line("13b", &a13);
    bytes_line("70b_slice", &a70);
    bytes_line("tiny", &tiny);

    /* argument errors, all detected on the host */
    {
        llama_model_args bad = tiny;
        bad.n_kv_heads = 3;
        check_line("kv_heads_not_dividing", llama_model_bytes(&bad, NULL, NULL, NULL, NULL, NULL));
        bad = tiny;
        bad.dtype = 7;
        check_line("unknown_dtype", llama_model_bytes(&bad, NULL, NULL, NULL, NULL, NULL));
        check_line("null_args", llama_model_bytes(NULL, NULL, NULL, NULL, NULL, NULL));
    }
    {
        llama_model* m = NULL;
        check_line("create_null_arena", llama_model_create(&tiny, NULL, (size_t)1 << 30, NULL, &m));
        check_line("create_left_null", m == NULL ? 0 : 1);
    }
    {
        int32_t tok = 0;
        float f = 0.0f;
        llama_sampling s;
        s.temperature = 0.7f;
        s.top_p = 0.9f;
        check_line("prefill_null_model", llama_prefill(NULL, &tok, NULL, 1, 1, 0, NULL, 0, NULL));
        check_line("decode_null_model", llama_decode_step(NULL, &tok, &tok, 1, &s, &f, &tok, NULL, 0, NULL));
        check_line("sample_no_uniforms", llama_sample(&f, 1, 10, 0.7f, 0.9f, NULL, &tok, NULL));
        check_line("logprobs_empty", llama_token_logprobs(&f, &tok, 0, 10, &f, NULL));
        check_line("op_linear_bad_dtype", llama_op_linear(&f, &f, 4, 128, 64, 7, &f, NULL, 0, NULL));
        check_line("status_null_model", llama_model_status(NULL, NULL));
    }
    printf("launches %llu\n", (unsigned long long)llama_launch_count());
    printf("done\n");
    return 0;
}
