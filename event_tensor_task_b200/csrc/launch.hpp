// launch.hpp — CUDA-side entry points of the C ABI (defined in megakernel.cu).
#pragma once
#include <string>
#include <vector>

#include "plan.hpp"

namespace mk {
mk_status dev_query(int* n_sm, int* smem_optin, int* device, std::string& err);
int smem_fixed_bytes();
mk_status dev_bind(Plan& p, void* ws, size_t bytes, void* stream, const std::vector<unsigned char>& image,
                   std::string& err);
mk_status dev_launch(Plan& p, const mk_step_args* a, void* stream, std::string& err);
mk_status dev_status(Plan& p, mk_device_status* st, std::string& err);
mk_status dev_reset(Plan& p, void* stream, std::string& err);
mk_status dev_launch_static(Plan& p, const mk_step_args* a, void* stream, std::string& err);
mk_status dev_launch_moe(Plan& p, const mk_moe_args* a, void* stream, std::string& err);
}  // namespace mk
